"""CPU oracle for the GPT training step.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py``; never by the product package.  See ``gpt_oracle`` for what it
computes and which passages of the pages each part follows.
"""
from .gpt_oracle import *  # noqa: F401,F403
