"""Build variants of the CUDA library that the default build does not cover
(CPU only: nvcc cross-compiles for sm_100a without a GPU).

The prefill kernel carries optional event-trace hooks (%globaltimer stamps of
each role's pipeline events, compiled in with -DLA_TRACE) that are used for
timeline analysis; this keeps that build compiling and exporting its hook.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

from long_context_fwd_b200 import build


def test_trace_build_compiles_and_exports_its_hook(tmp_path):
    nvcc = build.nvcc()
    if not (os.path.exists(nvcc) or shutil.which(nvcc)):
        pytest.skip("nvcc not available")
    so = str(tmp_path / "liblightning_attn_trace.so")
    cmd = [nvcc] + build.NVCC_FLAGS + ["-DLA_TRACE", "-o", so] + build.SOURCES
    subprocess.run(cmd, check=True, timeout=900)
    lib = ctypes.CDLL(so)
    assert hasattr(lib, "lightning_attn_set_trace")
    assert hasattr(lib, "lightning_attn_fwd")
