"""The C-ABI library loads without a GPU, exports every symbol include/*.h declares, and
rejects malformed arguments on the host before touching CUDA."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

from sparse_attention_token_04_b200 import binding
from sparse_attention_token_04_b200.build import LIB_PATH, ROOT, build


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB_PATH):
        build()
    return binding.lib()


def declared_functions():
    names = []
    for header in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(header).read()
        names += re.findall(r"DSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("dsa_indexer_prefill", "dsa_indexer_decode", "indexcache_run", "topk_overlap"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for name in names:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported
    # nothing else leaks out of the library's own code
    assert not [s for s in exported if s.startswith("_ZN3dsa")]


def test_status_strings_and_version(lib):
    assert binding.dsa_abi_version() == 1
    assert binding.status_string(0) == "ok"
    assert "invalid" in binding.status_string(1)
    assert binding.status_string(99) == "unknown status"


def test_host_validation_without_gpu(lib):
    nul = None
    # null inputs
    st = lib.dsa_indexer_prefill(nul, nul, nul, nul, nul, 16, 0, 16, 64, 128, 8, nul, nul, nul, 0, nul)
    assert st == binding.DSA_ERR_INVALID
    st = lib.dsa_indexer_decode(nul, nul, nul, nul, nul, 1, 64, nul, 1, nul, 1, 64, 128, 8, nul, nul,
                                nul, 0, nul)
    assert st == binding.DSA_ERR_INVALID
    # patterns: leading S, bad character, wrong length
    shape = binding.dsa_indexer_shape()
    arr = (binding.dsa_layer_inputs * 2)()
    fb = (ctypes.c_void_p * 1)(ctypes.c_void_p(16))
    out = (ctypes.c_void_p * 2)()
    for pat, n in ((b"SF", 2), (b"FX", 2), (b"FS", 3)):
        st = lib.indexcache_run(pat, n, ctypes.byref(shape), arr, fb, 1, out, binding.AFTER_LAYER_FN(),
                                None, None, 0, None)
        assert st == binding.DSA_ERR_INVALID, pat
    # decode: more requests than one launch takes, rejected before anything is enqueued
    fake = ctypes.c_void_p(1 << 20)
    st = lib.dsa_indexer_decode(fake, fake, fake, fake, fake, 1, 64, fake, 1, fake, 65536, 64, 128, 8,
                                fake, nul, nul, 0, nul)
    assert st == binding.DSA_ERR_UNSUPPORTED
    # overlap: too many layers / no pointers
    ptrs = (ctypes.c_void_p * 1)()
    assert lib.topk_overlap(ptrs, 65, 1, 1, 1, None, None, None, None, 0, None) == binding.DSA_ERR_INVALID
    # unsupported head shape is reported before any launch
    st = lib.dsa_prefill_workspace_bytes(16, 32, 128, 8)
    assert st == 0


def test_decode_workspace_size_matches_its_documented_layout(lib):
    """Header + [B][max_len] fp32 scores + [B][2048] u32 histograms + [B] 16-byte collection
    states + [B][8192] u64 candidate keys, sections 256-byte aligned; the no-alloc scratch is
    that workspace for the largest call it takes (34 MiB + 4352 B, as the header states)."""
    def align(x):
        return (x + 255) // 256 * 256

    for B, max_len in ((1, 64), (3, 640), (32, 200064), (256, 16384)):
        want = align(binding.DSA_WS_HEADER_BYTES + B * max_len * 4) + B * 2048 * 4
        want = align(want + B * 16) + B * 8192 * 8
        assert binding.dsa_decode_workspace_bytes(B, max_len, 64, 128, 2048) == want, (B, max_len)
    n_req, n_scores = binding.DSA_NOALLOC_MAX_REQUESTS, binding.DSA_NOALLOC_MAX_SCORES
    assert binding.dsa_decode_workspace_bytes(n_req, n_scores // n_req, 64, 128, 2048) == 34 * 2**20 + 4352


def test_sparse_attention_workspace_and_host_validation(lib):
    """The attention workspace is the header, then [B][topk/256][512][128] fp32 partials and
    [B][topk/256][2][128] fp32 row maxima and sums; unsupported shapes and malformed arguments
    are rejected on the host, before anything is enqueued."""
    for B, topk in ((1, 256), (3, 768), (32, 2048)):
        n_split = topk // 256
        want = binding.DSA_WS_HEADER_BYTES + B * n_split * 512 * 128 * 4 + B * n_split * 2 * 128 * 4
        assert lib.dsa_sparse_attention_workspace_bytes(B, topk) == want
    for B, topk in ((0, 256), (1, 0), (1, 300), (1, 2304)):
        assert lib.dsa_sparse_attention_workspace_bytes(B, topk) == 0

    p = ctypes.c_void_p(1 << 20)  # never dereferenced: every case below returns first
    f = lib.dsa_sparse_attention_decode

    def call(q=p, latent=p, n_blocks=4, block_size=64, table=p, max_blocks=4, seq=p, idx=p, B=2,
             Hq=128, dqk=576, dv=512, topk=256, scale=0.05, out=p, ws=None, ws_bytes=0):
        return f(q, latent, n_blocks, block_size, table, max_blocks, seq, idx, B, Hq, dqk, dv, topk,
                 scale, out, ws, ws_bytes, None)

    assert call(q=None) == binding.DSA_ERR_INVALID
    assert call(idx=None) == binding.DSA_ERR_INVALID
    assert call(B=0) == binding.DSA_ERR_INVALID
    assert call(scale=0.0) == binding.DSA_ERR_INVALID
    assert call(scale=float("nan")) == binding.DSA_ERR_INVALID
    assert call(q=ctypes.c_void_p((1 << 20) + 8)) == binding.DSA_ERR_INVALID   # not 16-byte aligned
    assert call(Hq=64) == binding.DSA_ERR_UNSUPPORTED
    assert call(dqk=512) == binding.DSA_ERR_UNSUPPORTED
    assert call(topk=300) == binding.DSA_ERR_UNSUPPORTED
    assert call(topk=4096) == binding.DSA_ERR_UNSUPPORTED
    assert call() == binding.DSA_ERR_INVALID                                   # no workspace
    need = lib.dsa_sparse_attention_workspace_bytes(2, 256)
    assert call(ws=p, ws_bytes=need - 1) == binding.DSA_ERR_INVALID            # too small
