// Host utilities: device properties, TMA tensor-map encoding, status strings.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <unordered_map>

#include "host.h"

namespace gpt {

thread_local int64_t g_launch_count = 0;

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("GPTSTEP_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

gpt_status device_info(int* num_sms) {
  static std::mutex mu;
  static int cached_sms[64] = {0};
  int dev = 0;
  GPT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPT_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (cached_sms[dev] == 0) {
    int major = 0, sms = 0;
    GPT_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    GPT_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    if (major != 10) return GPT_ERR_NO_DEVICE;
    cached_sms[dev] = sms;
  }
  *num_sms = cached_sms[dev];
  return GPT_OK;
}

static thread_local cudaError_t g_last_cuda_error = cudaSuccess;
void note_cuda_error(cudaError_t e) { g_last_cuda_error = e; }

gpt_status ensure_smem_limit(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // kernel -> bit per device
  int dev = 0;
  GPT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPT_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  uint64_t& mask = done[kernel];
  if (!((mask >> dev) & 1)) {
    GPT_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    mask |= 1ull << dev;
  }
  return GPT_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static bool encode_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank,
                       const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                       bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides_bytes[i];
  const CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_map_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                    swizzle128);
}

bool encode_map_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box, true);
}

bool encode_map_f32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, rank, dims, strides_bytes, box, false);
}

}  // namespace gpt

extern "C" const char* gpt_strerror(int status) {
  switch (status) {
    case GPT_OK: return "ok";
    case GPT_ERR_INVALID_ARG: return "invalid argument";
    case GPT_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or alignment";
    case GPT_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GPT_ERR_CUDA: return "CUDA runtime error";
    case GPT_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case GPT_ERR_TOKEN_OUT_OF_RANGE: return "token or target id out of range";
    case GPT_ERR_NO_DEVICE: return "no sm_100 device is current";
    case GPT_ERR_NUMERIC_RANGE: return "attention score bound out of the supported range";
    default: return "unknown status";
  }
}

extern "C" const char* gpt_last_cuda_error(void) {
  static thread_local char buf[256];
  const cudaError_t e = gpt::g_last_cuda_error;
  snprintf(buf, sizeof(buf), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return buf;
}
