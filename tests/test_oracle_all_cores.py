"""The all-core build of the oracle (oracle.c compiled with -fopenmp, used only
to time the oracle on every host core) gives the same bits as the default
single-threaded build: its pragmas only hand independent outputs and rows to
threads, each still computed by the same serial code."""
import os
import shutil

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")


def _bits(x):
    return np.ascontiguousarray(x).view(np.uint32)


def _both(fn):
    ref = fn()
    with oracle.library(oracle.build_all_cores()):
        par = fn()
    return ref, par


def test_gemm_tree_same_bits_on_all_cores():
    os.environ.setdefault("OMP_NUM_THREADS", "4")
    a = synth.normal_bf16(71, (37, 512), std=1.0)
    b = synth.normal_bf16(72, (512, 40), std=0.05)
    for T in (1, 4):
        (c0, s0), (c1, s1) = _both(lambda: oracle.gemm_tree(a, b, b_nk=False, T=T, leaf=32, shards=True))
        assert np.array_equal(_bits(c0), _bits(c1)), T
        assert np.array_equal(_bits(s0), _bits(s1)), T


def test_logprob_same_bits_on_all_cores():
    os.environ.setdefault("OMP_NUM_THREADS", "4")
    M, V, H = 9, 1000, 256
    h = synth.normal_bf16(73, (M, H), std=1.0)
    w = synth.normal_bf16(74, (V, H), std=0.2)
    t = synth.uniform_int32(75, M, 0, V)
    for noninv in (False, True):
        o0, o1 = _both(lambda: oracle.logprob(h, w, t, T=2, leaf=64, vpad=1024, noninv=noninv))
        assert np.array_equal(_bits(o0), _bits(o1)), noninv
