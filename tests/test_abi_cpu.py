"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/gecko.h declares, and rejects bad arguments on the
host before touching CUDA."""
import ctypes
import os
import re

import pytest

from long_context_sequence_sca_b200 import build as B
from long_context_sequence_sca_b200 import lib as L

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gecko.h")


@pytest.fixture(scope="module")
def so():
    B.build()
    return L.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gecko_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    assert set(declared_functions()) == set(L.EXPORTS)


def test_library_exports_every_declared_symbol(so):
    for name in declared_functions():
        assert hasattr(so, name), name
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_no_torch_types_in_header():
    text = open(HEADER).read()
    assert "torch" not in text.lower().replace("pytorch", "") and "at::" not in text


# Each case fails host validation, so nothing reaches CUDA.
FAKE = 0x100000  # 16-byte aligned, never dereferenced


def _call(ptrs=None, B=1, H=1, T=256, c=128, d=64, dtype=1):
    ptrs = ptrs or [FAKE] * 7
    return L.gecko_sca_awm_forward(*ptrs, B, H, T, c, d, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[0] + [FAKE] * 6), 1),
    (dict(dtype=7), 1),
    (dict(B=0), 1),
    (dict(T=-4), 1),
    (dict(d=96), 2),
    (dict(c=96, T=192), 2),
    (dict(T=300, c=128), 2),
    (dict(ptrs=[FAKE, FAKE + 8] + [FAKE] * 5), 3),
    (dict(B=1 << 40, H=1 << 20), 2),
    (dict(B=256, H=256), 2),                 # B*H above the grid limit
    (dict(T=64 * 65536, c=64), 2),           # T/c above the grid limit
])
def test_host_validation_rejects(so, kw, code):
    assert _call(**kw) == code
    assert L.gecko_last_error()


def test_state_query_rejects_null(so):
    assert L.gecko_awm_state(0, 0, 1, 1, 64, None) == 1


def _cema(ptrs=None, B=1, L=1000, D=64, h=16, dtype=1):
    ptrs = ptrs or [FAKE] * 7 + [0, 0, 0]
    return L_cema(ptrs, B, L, D, h, dtype)


def L_cema(ptrs, B, Lt, D, h, dtype):
    return L.gecko_cema_forward(*ptrs, B, Lt, D, h, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[FAKE, 0] + [FAKE] * 5 + [0, 0, 0]), 1),   # y NULL
    (dict(dtype=3), 1),
    (dict(L=0), 1),
    (dict(h=8), 2),                                         # h must be 16
    (dict(L=65536 * 256), 2),                               # more chunks than grid.y holds
    (dict(B=70000), 2),
    (dict(ptrs=[FAKE] * 7 + [FAKE + 4, 0, 0]), 3),          # reset misaligned
    (dict(ptrs=[FAKE] * 7 + [0, 0, FAKE + 8]), 3),          # state_out misaligned
])
def test_cema_host_validation_rejects(so, kw, code):
    assert _cema(**kw) == code
    assert L.gecko_last_error()


def _tdnorm(ptrs=None, B=1, Lt=100, D=64, G=4, b1=0.9, b2=0.99, eps=1e-5, dtype=1):
    ptrs = ptrs or [FAKE] * 4
    return L.gecko_tdnorm_forward(*ptrs, B, Lt, D, G, b1, b2, eps, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[FAKE, 0, FAKE, FAKE]), 1),
    (dict(dtype=5), 1),
    (dict(G=0), 1),
    (dict(b1=1.0), 1),
    (dict(b2=-0.1), 1),
    (dict(eps=-1.0), 1),
    (dict(D=60, G=4), 2),           # D / G = 15: not a multiple of 8
    (dict(D=64, G=3), 2),           # D % G != 0
    (dict(ptrs=[FAKE, FAKE, FAKE + 4, FAKE]), 3),
])
def test_tdnorm_host_validation_rejects(so, kw, code):
    assert _tdnorm(**kw) == code
    assert L.gecko_last_error()


def _bwd(ptrs=None, B=1, H=1, T=256, c=128, d=64, dtype=1):
    ptrs = ptrs or [FAKE] * 15
    return L.gecko_sca_awm_backward(*ptrs, B, H, T, c, d, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[FAKE] * 7 + [0] + [FAKE] * 7), 1),     # lse NULL
    (dict(ptrs=[FAKE] * 14 + [0]), 1),                 # dkm NULL
    (dict(ptrs=[FAKE] * 10 + [FAKE + 4] + [FAKE] * 4), 3),
    (dict(ptrs=[FAKE] * 6 + [FAKE + 8] + [FAKE] * 8), 3),   # residual misaligned
    (dict(d=32), 2),
    (dict(T=300), 2),
    (dict(dtype=2), 1),
])
def test_backward_host_validation_rejects(so, kw, code):
    assert _bwd(**kw) == code
    assert L.gecko_last_error()


def test_train_forward_rejects_bad_lse(so):
    assert L.gecko_sca_awm_forward_train(*[FAKE] * 7, 0, 0, 1, 1, 256, 128, 64, 1, None) == 1
    assert L.gecko_sca_awm_forward_train(*[FAKE] * 7, FAKE + 4, 0, 1, 1, 256, 128, 64, 1, None) == 3
    assert L.gecko_sca_awm_forward_train(*[FAKE] * 7, FAKE, FAKE + 8, 1, 1, 256, 128, 64, 1, None) == 3


@pytest.mark.parametrize("call,code", [
    (lambda: L.gecko_awm_segment_logsum(0, FAKE, 1, 1, 256, 128, 64, 1, None), 1),
    (lambda: L.gecko_awm_segment_logsum(FAKE, FAKE, 1, 1, 300, 128, 64, 1, None), 2),
    (lambda: L.gecko_awm_segment_maps(FAKE, FAKE, 0, FAKE, 1, 1, 256, 128, 64, 1, None), 1),
    (lambda: L.gecko_awm_segment_maps(FAKE, FAKE, FAKE, FAKE + 4, 1, 1, 256, 128, 64, 1, None), 3),
    (lambda: L.gecko_awm_cp_logz(0, 2, 0, FAKE, 1, 1, 64, None), 1),
    (lambda: L.gecko_awm_cp_logz(FAKE, 2, 2, FAKE, 1, 1, 64, None), 1),
    (lambda: L.gecko_awm_cp_logz(FAKE, 2, 1, FAKE, 1, 1, 96, None), 2),
    (lambda: L.gecko_awm_cp_state(FAKE, FAKE, 3, -1, FAKE, 1, 1, 64, None), 1),
    (lambda: L.gecko_awm_cp_state(FAKE, FAKE + 4, 3, 1, FAKE, 1, 1, 64, None), 3),
    (lambda: L.gecko_awm_cp_state(FAKE, FAKE, 0, 0, FAKE, 1, 1, 64, None), 1),
    (lambda: L.gecko_awm_cp_logz(FAKE, 2, 1, FAKE, 256, 256, 64, None), 2),
    (lambda: L.gecko_awm_cp_state(FAKE, FAKE, 2, 1, FAKE, 256, 256, 64, None), 2),
], ids=["logsum-null", "logsum-shape", "maps-null", "maps-align", "logz-null", "logz-rank", "logz-d",
        "state-rank", "state-align", "state-P", "logz-grid", "state-grid"])
def test_context_parallel_host_validation_rejects(so, call, code):
    assert call() == code
    assert L.gecko_last_error()


def _noalloc_bytes(BH, T, c, d):
    """Working memory of the no-allocation entry point as include/gecko.h
    states it: eleven regions, each rounded up to 256 bytes."""
    al = lambda x: (x + 255) // 256 * 256
    S, R = T // c, (128 if c % 128 == 0 else 64)
    regions = [8 * BH * (T // R) * d] + [4 * BH * S * d] * 4 + [4 * BH * S * d * d] * 2 + \
              [4 * BH * (S + 1) * d * d, 2 * BH * (S + 1) * d * d, 2 * BH * S * d * d, 4 * BH * S]
    return sum(al(r) for r in regions)


# (768, 256, 64): the boundary moves if the smallest region (the per-chunk
# flags) is left out of the count
@pytest.mark.parametrize("T,c,d", [(32768, 4096, 128), (65536, 512, 128), (8192, 256, 64), (4096, 64, 64),
                                   (768, 256, 64)])
def test_noalloc_limit_follows_the_documented_size(so, T, c, d):
    """The largest B*H whose documented working memory fits the fixed scratch
    is accepted on the host; one more (b, h) is rejected with GECKO_ERR_LIMIT
    before any CUDA call."""
    import torch
    limit = 80 << 20
    bh = 1
    while _noalloc_bytes(bh + 1, T, c, d) <= limit:
        bh += 1
    assert _noalloc_bytes(bh, T, c, d) <= limit < _noalloc_bytes(bh + 1, T, c, d)
    assert L.gecko_sca_awm_forward_noalloc(*([FAKE] * 7), 1, bh + 1, T, c, d, 1, None) == 8
    if not torch.cuda.is_available():
        # passes the size check and stops at the first CUDA call (no device here)
        assert L.gecko_sca_awm_forward_noalloc(*([FAKE] * 7), 1, bh, T, c, d, 1, None) == 5
