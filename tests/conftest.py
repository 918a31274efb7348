"""Shared pytest configuration.

Tests marked ``gpu`` need a B200 (sm_100a) and the built CUDA library; the
rest run on any host and cover the oracle, the host-side logic and the
library's exported symbols.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 GPU and the built library")


def pytest_sessionstart(session):
    # The CUDA library and the oracle are built in-tree; (re)build them if a
    # source is newer than the binary so that every test sees current code.
    from tensor_core_gemm_fp16_b200 import build as tg_build
    import oracle

    tg_build.build()
    oracle.build()
