"""The C ABI library loads, exports every declared entry point, and rejects
bad arguments on the host (no GPU needed: none of these calls reaches a
kernel)."""
import ctypes as C
import os
import re

import pytest

import quantized_moe_expert_warp_b200 as mq
from quantized_moe_expert_warp_b200 import build as mqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    mqbuild.build()
    return mq.lib()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "moeq4.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ["moe_route", "moe_permute", "moe_expert_ffn_q4", "moe_combine", "moe_layer_forward",
              "moe_router_logits", "moe_router_workspace_size", "moe_pack_weights", "moe_layer_workspace_size", "moe_read_status"]:
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_binding_names_match_header():
    for n in declared_functions():
        assert hasattr(mq, n), n


def test_binding_constants_match_header():
    txt = open(os.path.join(ROOT, "include", "moeq4.h")).read()
    defs = dict(re.findall(r"#define (MOE_[A-Z0-9_]+) \(?(-?\d+)\)?", txt))
    assert len(defs) >= 9
    for name, value in defs.items():
        py = name.replace("MOE_WFMT_", "WFMT_")
        assert getattr(mq, py) == int(value), name
    # the ctypes structs mirror the header's field order
    for struct, fields in (("moe_config_t", mq.Config._fields_), ("moe_layer_t", mq.Layer._fields_),
                           ("moe_debug_t", mq.Debug._fields_)):
        block = txt[:txt.index("} " + struct + ";")]
        block = block[block.rindex("typedef struct"):]
        names = re.findall(r"\b(\w+)\s*;", re.sub(r"/\*.*?\*/", "", block, flags=re.S))
        assert names == [f[0] for f in fields], (struct, names)


def cfg(**kw):
    d = dict(H=2048, I=512, E=256, k=8, G=128, has_shared=1, renorm=1, wfmt=mq.WFMT_INT4_SYM)
    d.update(kw)
    return mq.Config(**d)


def test_version(L):
    assert L.moe_version() >= 1


def test_packed_sizes_a3b(L):
    sz = [C.c_size_t() for _ in range(4)]
    assert L.moe_packed_sizes(C.byref(cfg()), *[C.byref(s) for s in sz]) == 0
    gu_q, gu_m, dn_q, dn_m = (s.value for s in sz)
    assert gu_q == 257 * 1024 * 2048 // 2
    assert dn_q == 257 * 2048 * 512 // 2
    assert gu_m == 257 * 1024 * (2048 // 128) * 2
    assert dn_m == 257 * 2048 * (512 // 128) * 2
    # 1,622,016 bytes per expert
    assert (gu_q + gu_m + dn_q + dn_m) // 257 == 1622016


def test_packed_sizes_q4k(L):
    sz = [C.c_size_t() for _ in range(4)]
    assert L.moe_packed_sizes(C.byref(cfg(wfmt=mq.WFMT_Q4K, G=256)), *[C.byref(s) for s in sz]) == 0
    total = sum(s.value for s in sz)
    assert total // 257 == 3 * 2048 * 512 // 256 * 144   # 144 bytes per 256 weights


@pytest.mark.parametrize("bad,code", [
    (dict(H=2000), mq.MOE_ERR_UNSUPPORTED),
    (dict(I=100), mq.MOE_ERR_UNSUPPORTED),
    (dict(k=0), mq.MOE_ERR_INVALID_ARG),
    (dict(k=40), mq.MOE_ERR_UNSUPPORTED),
    (dict(E=4, k=5), mq.MOE_ERR_UNSUPPORTED),
    (dict(G=48), mq.MOE_ERR_UNSUPPORTED),
    (dict(G=96), mq.MOE_ERR_UNSUPPORTED),
    (dict(G=16), mq.MOE_ERR_UNSUPPORTED),
    (dict(wfmt=7), mq.MOE_ERR_UNSUPPORTED),
    (dict(wfmt=mq.WFMT_Q4K, I=384), mq.MOE_ERR_UNSUPPORTED),
])
def test_config_validation(L, bad, code):
    sz = C.c_size_t()
    assert L.moe_packed_sizes(C.byref(cfg(**bad)), C.byref(sz), None, None, None) == code
    assert L.moe_last_error()
    assert L.moe_layer_workspace_size(C.byref(cfg(**bad)), 16) == 0


def test_workspace_sizes_grow_with_T(L):
    c = cfg()
    a = L.moe_layer_workspace_size(C.byref(c), 512)
    b = L.moe_layer_workspace_size(C.byref(c), 8192)
    assert 0 < a < b
    # intermediates at T = 8192: y_perm + shared_out alone are (8 + 1) * 8192 * 2048 * 2 bytes
    assert b > 9 * 8192 * 2048 * 2
    assert L.moe_permute_workspace_size(8192, 256, 8) > 0
    assert L.moe_expert_ffn_workspace_size(C.byref(c), 8192) > 0


def test_null_and_misaligned_pointers_are_rejected(L):
    assert L.moe_route(None, 4, 16, 2, 1, None, None, None) == mq.MOE_ERR_INVALID_ARG
    assert b"logits" in L.moe_last_error()
    assert L.moe_route(0x1001, 4, 16, 2, 1, 0x2000, 0x3000, None) == mq.MOE_ERR_INVALID_ARG
    assert b"aligned" in L.moe_last_error()
    assert L.moe_route(0x1000, 4, 16, 0, 1, 0x2000, 0x3000, None) == mq.MOE_ERR_INVALID_ARG
    assert L.moe_route(0x1000, 4, 16, 33, 1, 0x2000, 0x3000, None) == mq.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, None, None, None, None, 4, 2048, 8, None, None) == mq.MOE_ERR_INVALID_ARG
    assert L.moe_combine(0x1000, 0x1000, 0x1000, None, None, 4, 2044, 8, 0x1000, None) == mq.MOE_ERR_INVALID_ARG


def test_workspace_too_small_is_reported(L):
    need = L.moe_permute_workspace_size(64, 16, 2)
    rc = L.moe_permute(0x1000, 64, 16, 2, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, need - 16, None)
    assert rc == mq.MOE_ERR_WORKSPACE
    layer = mq.Layer(cfg(), 0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    rc = L.moe_layer_forward(C.byref(layer), 0x1000, 512, 0x1000, 0x1000, 1024, None, None)
    assert rc == mq.MOE_ERR_WORKSPACE
    # the router's split-K partials: several MB at T = 512
    rneed = L.moe_router_workspace_size(C.byref(cfg()), 512)
    assert rneed >= 8 * 512 * 256 * 4
    rc = L.moe_router_logits(C.byref(layer), 0x1000, 512, 0x1000, None, 0x1000, rneed - 16, None)
    assert rc == mq.MOE_ERR_WORKSPACE


def test_chunked_layer_checks_chunk_and_workspace(L):
    layer = mq.Layer(cfg(), 0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    rc = L.moe_layer_forward_chunked(C.byref(layer), 0x1000, 16000, 0x1000, 0, 0x1000, 1 << 40, None)
    assert rc == mq.MOE_ERR_INVALID_ARG and b"chunk" in L.moe_last_error()
    # the workspace has to hold one chunk, not all T tokens
    one = L.moe_layer_workspace_size(C.byref(cfg()), 8192)
    assert one < L.moe_layer_workspace_size(C.byref(cfg()), 16000)
    rc = L.moe_layer_forward_chunked(C.byref(layer), 0x1000, 16000, 0x1000, 8192, 0x1000, one - 256, None)
    assert rc == mq.MOE_ERR_WORKSPACE


def test_layer_rejects_missing_shared_gate(L):
    layer = mq.Layer(cfg(), 0x1000, None, None, 0x1000, 0x1000, 0x1000, 0x1000)
    need = L.moe_layer_workspace_size(C.byref(cfg()), 512)
    rc = L.moe_layer_forward(C.byref(layer), 0x1000, 512, 0x1000, 0x1000, need, None, None)
    assert rc == mq.MOE_ERR_INVALID_ARG
    assert b"shared_gate" in L.moe_last_error()


def test_zero_tokens_is_a_no_op(L):
    layer = mq.Layer(cfg(), 0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    need = L.moe_layer_workspace_size(C.byref(cfg()), 0)
    assert L.moe_layer_forward(C.byref(layer), None, 0, None, 0x1000, need, None, None) == 0
    assert L.moe_route(None, 0, 16, 2, 1, None, None, None) == 0


def test_binding_refuses_host_and_strided_tensors(L):
    torch = pytest.importorskip("torch")
    logits = torch.zeros((4, 16), dtype=torch.float32)
    ids = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mq.moe_route(logits, 4, 16, 2, True, ids, ids.float(), stream=0)

    class FakeCuda:
        is_cuda = True

        def is_contiguous(self):
            return False

        def stride(self):
            return (1, 4)

    with pytest.raises(ValueError, match="contiguous"):
        mq.moe_route(FakeCuda(), 4, 16, 2, True, 0x1000, 0x1000, stream=0)


def test_decode_admission_and_workspace(L):
    c = cfg()
    # a3b shape: T = 1..8 admitted, 9 and more go through moe_layer_forward
    sizes = [L.moe_layer_decode_workspace_size(C.byref(c), t) for t in (1, 2, 8)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    # h in bf16 for T k + T pairs (the expert outputs never leave shared memory)
    assert sizes[2] >= (8 * 8 + 8) * 512 * 2
    assert L.moe_layer_decode_workspace_size(C.byref(c), 9) == 0
    layer = mq.Layer(c, 0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    rc = L.moe_layer_decode(C.byref(layer), 0x1000, 9, 0x1000, 0x1000, 1 << 30, None, None)
    assert rc == mq.MOE_ERR_UNSUPPORTED and b"8 tokens" in L.moe_last_error()
    rc = L.moe_layer_decode(C.byref(layer), 0x1000, 4, 0x1000, 0x1000,
                            L.moe_layer_decode_workspace_size(C.byref(c), 4) - 256, None, None)
    assert rc == mq.MOE_ERR_WORKSPACE
    # the intermediates of 8 tokens at k = 32, I = 1024 do not fit in shared memory (1 token does)
    big = cfg(k=32, I=1024)
    assert L.moe_layer_decode_workspace_size(C.byref(big), 8) == 0
    assert L.moe_layer_decode_workspace_size(C.byref(big), 1) > 0
    layer = mq.Layer(big, 0x1000, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    rc = L.moe_layer_decode(C.byref(layer), 0x1000, 8, 0x1000, 0x1000, 1 << 30, None, None)
    assert rc == mq.MOE_ERR_UNSUPPORTED and b"shared memory" in L.moe_last_error()
    # zero tokens: nothing to do
    assert L.moe_layer_decode(C.byref(layer), None, 0, None, 0x1000, 1 << 20, None, None) == mq.MOE_OK
