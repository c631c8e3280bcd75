"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and its host-only logic (sizes, argument checks, seeds) is right."""
import ctypes
import os
import re

import pytest

import decode_matmul_b200 as tq
import oracle
import tqsynth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^TQ_API\s+[\w\s\*]+?\b(tq_\w+)\(", txt, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 15
    L = tq.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(tq.EXPORTS) <= set(names)


@pytest.mark.parametrize("n,k", [(1024, 1024), (4096, 2560), (1024, 2560), (2560, 4096), (9728, 2560),
                                 (2560, 9728), (14336, 4096), (4096, 14336), (6144, 5120), (5120, 6144),
                                 (17408, 5120), (5120, 17408)])
def test_pack_info_size_invariant(n, k):
    info = tq.tq_pack_info(n, k)
    assert info["packed_bytes"] * 128 == n * k * 33
    assert info["packed_bytes"] == tqsynth.pack_bytes(n, k)
    assert info["bits_per_weight"] == 2.0625
    assert (info["group"], info["block"], info["rht_block"], info["n_states"]) == (4, 256, 512, 8)
    assert info["codebook_bytes"] == 16384
    c = tqsynth.codes(0, 0, 0, 2, k)
    assert c.nbytes // 2 * n == info["code_bytes"]


def test_pack_info_rejects_bad_shapes():
    for n, k in [(0, 512), (-1, 512), (16, 0), (16, 256), (16, 1000), (16, -512)]:
        with pytest.raises(tq.TqError) as e:
            tq.tq_pack_info(n, k)
        assert e.value.status == tq.TQ_ERR_SHAPE
    assert tq.lib().tq_pack_info(16, 512, None) == tq.TQ_ERR_NULL


def test_stack_workspace_sizes_monotone():
    assert tq.tq_gemv_workspace(1024, 1024) > 0
    assert tq.tq_gemm_workspace(1024, 1024, 64) >= tq.tq_gemm_workspace(1024, 1024, 1)
    with pytest.raises(tq.TqError):
        tq.tq_gemm_workspace(1024, 1024, 5000)


def _fake_layer(hidden, q, kv, inter):
    """A tq_layer_t of fake (aligned, never dereferenced) pointers."""
    def w(n, k):
        return tq.tq_weight_t(16, 16, 16, n, k)
    return tq.tq_layer_t(w(q, hidden), w(kv, hidden), w(kv, hidden), w(hidden, q), w(inter, hidden),
                         w(inter, hidden), w(hidden, inter))


def test_stack_output_offsets():
    """Host-side layout only: per-phase output buffers up to 16 tokens (the
    persistent kernels), one shared buffer beyond; the down outputs are where
    tq_layer_stack_buffers says."""
    layers = [_fake_layer(1024, 1536, 200, 2560)] * 3
    o1 = tq.tq_layer_stack_outputs(layers, 1)
    assert len(set(o1)) == 4 and all(o % 256 == 0 for o in o1)
    assert o1[3] == tq.tq_layer_stack_buffers(layers, 1)[4]
    # each buffer holds the widest phase (gate|up: 2 x 2560 fp32 rows) without overlap
    sizes = sorted(o1)
    assert all(b - a >= 4 * 2 * 2560 for a, b in zip(sizes, sizes[1:]))
    assert max(o1) + 4 * 2 * 2560 <= tq.tq_layer_stack_workspace(layers, 1)
    o4 = tq.tq_layer_stack_outputs(layers, 16)
    assert len(set(o4)) == 4 and o4[3] == tq.tq_layer_stack_buffers(layers, 16)[4]
    o32 = tq.tq_layer_stack_outputs(layers, 32)
    assert len(set(o32)) == 1 and o32[0] == tq.tq_layer_stack_buffers(layers, 32)[4]
    with pytest.raises(tq.TqError):
        tq.tq_layer_stack_outputs([_fake_layer(1024, 1536, 200, 2000)], 1)  # gate.n not a multiple of 512


def test_argument_checks_before_any_device_call():
    L = tq.lib()
    W = tq.tq_weight_t(16, 16, 16, 32, 512)  # fake, aligned addresses; never dereferenced
    # shape errors
    bad = tq.tq_weight_t(16, 16, 16, 32, 500)
    assert L.tq_gemv(ctypes.byref(bad), 16, 16, 16, 1 << 20, None) == tq.TQ_ERR_SHAPE
    assert L.tq_gemm(ctypes.byref(W), 16, -1, 16, 16, 1 << 20, None) == tq.TQ_ERR_SHAPE
    assert L.tq_rht(16, 1, 500, 0, 16, tq.TQ_F32, None) == tq.TQ_ERR_SHAPE
    assert L.tq_rht(16, 1, 512, 0, 16, 7, None) == tq.TQ_ERR_SHAPE
    # null / alignment
    assert L.tq_gemv(None, 16, 16, 16, 1 << 20, None) == tq.TQ_ERR_NULL
    assert L.tq_gemv(ctypes.byref(W), None, 16, 16, 1 << 20, None) == tq.TQ_ERR_NULL
    assert L.tq_gemv(ctypes.byref(W), 18, 16, 16, 1 << 20, None) == tq.TQ_ERR_ALIGN
    mis = tq.tq_weight_t(17, 16, 16, 32, 512)
    assert L.tq_decode(ctypes.byref(mis), 16, None) == tq.TQ_ERR_ALIGN
    assert L.tq_rht(18, 1, 512, 0, 16, tq.TQ_F32, None) == tq.TQ_ERR_ALIGN
    # empty work is fine and launches nothing
    assert L.tq_rht(16, 0, 512, 0, 16, tq.TQ_F32, None) == tq.TQ_OK
    assert L.tq_gemm(ctypes.byref(W), 16, 0, 16, 16, 1 << 20, None) == tq.TQ_OK


def test_gemv_k_limit_and_new_entry_points_checks():
    L = tq.lib()
    past = tq.tq_weight_t(16, 16, 16, 32, tq.TQ_GEMV_MAX_K + 512)
    # one 512-block past the batch-1 shared-memory limit: refused before any device call
    assert L.tq_gemv(ctypes.byref(past), 16, 16, 16, 1 << 30, None) == tq.TQ_ERR_SHAPE
    assert L.tq_gemv_noalloc(ctypes.byref(past), 16, 16, None) == tq.TQ_ERR_SHAPE
    assert tq.TQ_GEMV_MAX_K % 512 == 0 and 16384 + 4 * tq.TQ_GEMV_MAX_K <= 227 * 1024
    assert 16384 + 4 * (tq.TQ_GEMV_MAX_K + 512) > 227 * 1024
    # status query
    v = ctypes.c_int32()
    assert L.tq_workspace_status(None, ctypes.byref(v), None) == tq.TQ_ERR_NULL
    assert L.tq_workspace_status(16, None, None) == tq.TQ_ERR_NULL
    # stack options: a negative block index other than -1 is refused first
    layers = [_fake_layer(1024, 1536, 256, 2560)]
    arr = (tq.tq_layer_t * 1)(*layers)
    opt = tq.tq_stack_options_t(0, -2)
    assert L.tq_layer_stack_ex(arr, 1, 16, 1, 0, 16, 16, 1 << 30, ctypes.byref(opt), None) == tq.TQ_ERR_VALUE
    w = tq.tq_weight_t(16, 16, 16, 1024, 1536)
    assert L.tq_gemm_ex(ctypes.byref(w), 16, 64, 16, 16, 1 << 30, ctypes.byref(opt), None) == tq.TQ_ERR_VALUE


def test_gemm_workspace_covers_split_partials():
    # the tcgen05 kernel's split-k partial sums ([tiles][splits][BN][128]
    # fp32) live in the workspace after the 64 KB counter region; the query
    # must cover the largest split the launcher can choose: 148 CTAs, or 296
    # (two per SM) at 64-token tiles, and never more splits than 256-weight
    # blocks
    for n, k, m in [(5120, 17408, 48), (8192, 5120, 64), (2560, 9728, 64), (1040, 1536, 64), (2560, 4096, 512),
                    (6144, 2560, 512), (128, 512, 200)]:
        bn = 64 if m <= 64 else (128 if m <= 128 else 256)
        tiles = -(-n // 128) * -(-m // bn)
        blocks = k // 256
        splits = min(max(1, (296 if bn == 64 else 148) // tiles), blocks)
        need = 64 * 1024 + tiles * splits * bn * 128 * 4
        assert tq.tq_gemm_workspace(n, k, m) >= need, (n, k, m)


def test_stack_phase_seed_matches_oracle():
    # both sides implement SplitMix64 from its published definition
    for s, l, p in [(0, 0, 0), (0, 35, 3), (12345, 7, 2), (2 ** 64 - 1, 63, 1)]:
        assert tq.tq_stack_phase_seed(s, l, p) == oracle.stack_phase_seed(s, l, p)


def test_status_strings():
    for st in range(10):
        assert len(tq.lib().tq_status_string(st)) > 0
    assert tq.lib().tq_status_string(99) == b"unknown status"


def test_encode_argument_checks():
    L = tq.lib()
    f = ctypes.c_float
    ok = dict(w=16, n=4, k=512, cb=16, gain=f(1.0), refits=1, codes=16, scales=16, err=16)

    def call(**kw):
        a = dict(ok, **kw)
        return L.tq_encode(a["w"], a["n"], a["k"], a["cb"], a["gain"], a["refits"], a["codes"], a["scales"],
                           a["err"], None)

    for n, k in [(0, 512), (4, 256), (4, 0), (4, 768)]:
        assert call(n=n, k=k) == tq.TQ_ERR_SHAPE
    for g in [0.0, -1.0, float("inf"), float("nan")]:
        assert call(gain=f(g)) == tq.TQ_ERR_VALUE
    assert call(refits=-1) == tq.TQ_ERR_VALUE
    assert call(refits=tq.TQ_ENCODE_MAX_REFITS + 1) == tq.TQ_ERR_VALUE
    for name in ("w", "cb", "codes", "scales"):
        assert call(**{name: None}) == tq.TQ_ERR_NULL
    for name, v in (("w", 20), ("cb", 24), ("codes", 40), ("scales", 18), ("err", 22)):
        assert call(**{name: v}) == tq.TQ_ERR_ALIGN


def test_ldlq_argument_checks():
    L = tq.lib()
    f = ctypes.c_float
    need = tq.tq_ldlq_workspace(4, 512)
    assert need == 4 * (512 + 256) * 4
    ok = dict(w=16, n=4, k=512, u=16, cb=16, gain=f(1.0), refits=1, codes=16, scales=16, err=None, ws=16,
              wsb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return L.tq_ldlq_encode(a["w"], a["n"], a["k"], a["u"], a["cb"], a["gain"], a["refits"], a["codes"],
                                a["scales"], a["err"], a["ws"], a["wsb"], None)

    assert call(k=768) == tq.TQ_ERR_SHAPE
    assert call(gain=f(-2.0)) == tq.TQ_ERR_VALUE
    assert call(u=None) == tq.TQ_ERR_NULL
    assert call(u=24) == tq.TQ_ERR_ALIGN
    assert call(ws=None) == tq.TQ_ERR_WORKSPACE
    assert call(wsb=need - 1) == tq.TQ_ERR_WORKSPACE
    assert call(ws=20) == tq.TQ_ERR_ALIGN

