"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
function include/kda.h declares, and rejects bad arguments before enqueuing work.
Every call below breaks exactly one rule that is checked before any launch."""
import os
import re

import pytest

import gated_delta_rule_85_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, CUDA, WORKSPACE = 0, -1, -2, -3, -4, -5


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_85_b200.build import build
    build()
    return kda.load_library()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "kda_chunk_forward" in names and "kda_recurrent_step" in names
    for name in names:
        assert hasattr(lib, name), f"libkda.so does not export {name}"
    assert lib.kda_api_version() == 1


# fake but 256-byte aligned "device" addresses: never dereferenced, every call fails validation
A = [0x10000 * (i + 1) for i in range(12)]


def prefill(lib, **over):
    a = dict(q=A[0], k=A[1], v=A[2], g=A[3], b=A[4], s0=A[5], o=A[6], fs=A[7], cu=None,
             B=1, T=128, H=2, dk=128, dv=128, N=1, dtype=0, chunk=64, ws=A[8], wsb=1 << 20, st=None)
    a.update(over)
    return lib.kda_chunk_forward(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["o"], a["fs"], a["cu"],
                                 a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dtype"], a["chunk"],
                                 a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), INVALID),
    (dict(o=None), INVALID),
    (dict(beta_missing=True), INVALID),
    (dict(T=-1), INVALID),
    (dict(H=0), INVALID),
    (dict(N=2), INVALID),                       # N != B without cu_seqlens
    (dict(cu=A[9], B=2, N=2), INVALID),         # packed input needs B == 1
    (dict(dk=96), UNSUPPORTED),
    (dict(dv=256), UNSUPPORTED),
    (dict(chunk=32), UNSUPPORTED),
    (dict(dtype=7), UNSUPPORTED),
    (dict(q=A[0] + 8), MISALIGNED),
    (dict(fs=A[7] + 4), MISALIGNED),
    (dict(b=A[4] + 2), MISALIGNED),
])
def test_prefill_rejects(lib, over, code):
    if over.pop("beta_missing", False):
        over["b"] = None
    assert prefill(lib, **over) == code
    assert lib.kda_last_error().decode() != ""


def test_simt_rejects(lib):
    rc = lib.kda_chunk_forward_simt(A[0], A[1], A[2], A[3], A[4], None, A[6], None, None,
                                    1, 64, 1, 64, 48, 1, 1, 64, None)
    assert rc == UNSUPPORTED


def step(lib, **over):
    a = dict(q=A[0], k=A[1], v=A[2], g=A[3], b=A[4], s=A[5], o=A[6], N=4, H=2, dk=128, dv=128, dtype=0, st=None)
    a.update(over)
    return lib.kda_recurrent_step(a["q"], a["k"], a["v"], a["g"], a["b"], a["s"], a["o"], a["N"], a["H"],
                                  a["dk"], a["dv"], a["dtype"], a["st"])


@pytest.mark.parametrize("over,code", [
    (dict(s=None), INVALID),
    (dict(N=-1), INVALID),
    (dict(dk=32), UNSUPPORTED),
    (dict(dtype=3), UNSUPPORTED),
    (dict(s=A[5] + 4), MISALIGNED),
    (dict(v=A[2] + 2), MISALIGNED),
])
def test_step_rejects(lib, over, code):
    assert step(lib, **over) == code


def test_empty_work_is_a_no_op(lib):
    assert step(lib, N=0) == OK


def test_status_requires_pointer(lib):
    assert lib.kda_get_device_status(None, 0, None) == INVALID


REC128, REC64 = 58368, 33792   # two-pass workspace bytes per (chunk slot, head) at dk = 128 / 64


def two_pass_ws(slots, H, rec):
    """One record per (chunk slot, head)."""
    return slots * H * rec


def test_workspace_sizes(lib):
    f = lib.kda_chunk_forward_workspace_size_ex
    FUSED, TWO_PASS, AUTO = 1, 2, 0
    # slots = ceil(B*T / 64) + num_seqs
    assert f(1, 8192, 32, 128, 128, 1, 0, 64, TWO_PASS) == two_pass_ws(128 + 1, 32, REC128)
    assert f(1, 8192, 32, 128, 128, 1, 0, 64, FUSED) == 0
    assert f(1, 8192, 32, 128, 128, 1, 0, 64, AUTO) == two_pass_ws(128 + 1, 32, REC128)     # 32 chains: two-pass
    assert f(1, 1 << 20, 32, 128, 128, 22, 0, 64, AUTO) == 0                         # 704 chains: fused
    assert f(2, 1 << 19, 8, 128, 128, 2, 0, 64, AUTO) == 0      # two sequences over AUTO's 1 GiB: fused
    assert f(3, 100, 2, 64, 64, 3, 0, 64, TWO_PASS) == two_pass_ws(5 + 3, 2, REC64)
    assert f(1, 100, 2, 64, 64, 1, 1, 64, TWO_PASS) == 0                             # fp32 path
    assert f(2, 0, 2, 128, 128, 2, 0, 64, TWO_PASS) == 0                             # no tokens
    assert lib.kda_chunk_forward_workspace_size(1, 8192, 32, 128, 128, 1, 0, 64) == two_pass_ws(128 + 1, 32, REC128)


def windowed_ws(H, dk, dv, rec, limit):
    """AUTO's windowed two-pass workspace: two fp32 [H][dk][dv] carry states (rounded
    up to 1 KiB) and the records of the longest window that fits `limit`, plus the
    one slack slot a sequence has."""
    carry = -(-2 * H * dk * dv * 4 // 1024) * 1024
    chunks = (limit - carry) // (H * rec) - 1
    return carry + (chunks + 1) * H * rec


def test_auto_workspace_budget(lib):
    f = lib.kda_chunk_forward_workspace_size_ex
    TWO_PASS, AUTO = 2, 0
    GiB = 1 << 30
    assert lib.kda_set_auto_workspace_limit(0) == GiB        # the default, left in place
    # prefill_128k: 2049 slots x 32 heads x 58368 B = 3.8 GB unwindowed, <= 1 GiB windowed
    assert f(1, 131072, 32, 128, 128, 1, 0, 64, TWO_PASS) == two_pass_ws(2048 + 1, 32, REC128)
    w = f(1, 131072, 32, 128, 128, 1, 0, 64, AUTO)
    assert w == windowed_ws(32, 128, 128, REC128, GiB)
    assert GiB - 32 * REC128 < w <= GiB
    assert f(1, 1 << 20, 8, 128, 128, 1, 0, 64, AUTO) == windowed_ws(8, 128, 128, REC128, GiB)
    # a smaller budget: small inputs go windowed too; multi-sequence inputs go fused
    limit = 2 << 20   # windows of 320 tokens at H=4, dk=dv=128; 832 at dk=dv=64
    try:
        assert lib.kda_set_auto_workspace_limit(limit) == GiB
        assert f(1, 1000, 4, 128, 128, 1, 0, 64, AUTO) == windowed_ws(4, 128, 128, REC128, limit)
        assert f(1, 1000, 4, 64, 64, 1, 0, 64, AUTO) == windowed_ws(4, 64, 64, REC64, limit)
        assert f(1, 100, 4, 128, 128, 1, 0, 64, AUTO) == two_pass_ws(2 + 1, 4, REC128)   # fits: one pair
        assert f(2, 1000, 4, 128, 128, 2, 0, 64, AUTO) == 0
        assert f(1, 1000, 4, 128, 128, 1, 0, 64, TWO_PASS) == two_pass_ws(16 + 1, 4, REC128)
        # a budget below one window's carry and record: fused
        lib.kda_set_auto_workspace_limit(4096)
        assert f(1, 1000, 4, 128, 128, 1, 0, 64, AUTO) == 0
    finally:
        lib.kda_set_auto_workspace_limit(0)
    assert lib.kda_set_auto_workspace_limit(0) == GiB


def prefill_ex(lib, algo, ws, wsb):
    return lib.kda_chunk_forward_ex(A[0], A[1], A[2], A[3], A[4], A[5], A[6], A[7], None,
                                    1, 128, 2, 128, 128, 1, 0, 64, algo, ws, wsb, None)


def test_prefill_ex_rejects(lib):
    need = two_pass_ws(2 + 1, 2, REC128)
    assert prefill_ex(lib, 7, A[8], need) == INVALID            # unknown algo
    assert prefill_ex(lib, 2, A[8], need - 1) == WORKSPACE      # workspace too small
    assert prefill_ex(lib, 2, None, 0) == WORKSPACE             # workspace missing
    assert prefill_ex(lib, 2, A[8] + 16, need) == MISALIGNED    # workspace below 256-byte alignment


def test_static_ws_capacity_matches_header():
    """The binding's copy of KDA_STATIC_WS_BYTES equals the header's definition."""
    src = open(HEADER).read()
    m = re.search(r"#define\s+KDA_STATIC_WS_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", src)
    assert m, "KDA_STATIC_WS_BYTES definition not found"
    assert kda.STATIC_WS_BYTES == int(m.group(1)) << int(m.group(2))


def test_slot_entry_points_reject(lib):
    pre = lambda slots, num_slots, align=0: lib.kda_chunk_forward_slots(
        A[0], A[1], A[2], A[3], A[4], A[5], slots, A[6], None, 1, 128, 2, 128, 128, 1, num_slots, 0, 64, 0,
        A[8], 1 << 24, None)
    assert pre(None, 4) == INVALID                 # slot table missing
    assert pre(A[9], 0) == INVALID                 # empty pool
    assert pre(A[9] + 2, 4) == MISALIGNED          # slot table below 4-byte alignment
    dec = lambda slots, num_slots: lib.kda_recurrent_step_slots(
        A[0], A[1], A[2], A[3], A[4], A[5], slots, A[6], 4, 2, 128, 128, num_slots, 0, None)
    assert dec(None, 8) == INVALID
    assert dec(A[9], 0) == INVALID
    assert dec(A[9] + 1, 8) == MISALIGNED
    assert lib.kda_recurrent_step_slots(A[0], A[1], A[2], A[3], A[4], A[5], A[9], A[6], 0, 2, 128, 128, 8, 0,
                                        None) == OK   # no sequences: nothing to do


# backward workspace per (chunk slot, head), fp32: the chunk record (3 [64][dk]
# + 5 [64][64] + [dk][64] + dk, rows padded by 4 floats), the state at the chunk's
# start and the adjoint at its end ([dk][dv] each), and the column sums
# (3 [64][dk] + 2 [64][64] + 64 + dk)
def bwd_ws(slots, H, dk, dv):
    rec = 3 * 64 * (dk + 4) + 5 * 64 * 68 + dk * 68 + dk
    part = 3 * 64 * dk + 2 * 64 * 64 + 64 + dk
    return slots * H * (rec + 2 * dk * dv + part) * 4


def test_backward_workspace_sizes(lib):
    f = lib.kda_chunk_backward_workspace_size
    assert f(1, 8192, 32, 128, 128, 1) == bwd_ws(129, 32, 128, 128)
    assert f(3, 100, 2, 64, 64, 3) == bwd_ws(5 + 3, 2, 64, 64)
    assert f(1, 100, 2, 128, 64, 1) == bwd_ws(2 + 1, 2, 128, 64)
    assert f(2, 0, 2, 128, 128, 2) == 0          # no tokens
    assert f(1, 100, 2, 96, 128, 1) == 0         # unsupported dk


UNIT128 = 148480   # tensor-core backward bytes per (chunk slot, head) at dk = dv = 128
BWD_AUTO, BWD_TENSOR, BWD_SIMT = 0, 1, 2


def test_backward_workspace_sizes_by_schedule(lib):
    f = lib.kda_chunk_backward_workspace_size_ex
    assert f(1, 8192, 32, 128, 128, 1, 0, BWD_AUTO) == 129 * 32 * UNIT128     # bf16, dk = dv = 128: tensor cores
    assert f(1, 8192, 32, 128, 128, 1, 0, BWD_TENSOR) == 129 * 32 * UNIT128
    assert f(1, 8192, 32, 128, 128, 1, 0, BWD_SIMT) == bwd_ws(129, 32, 128, 128)
    assert f(1, 8192, 32, 128, 128, 1, 1, BWD_AUTO) == bwd_ws(129, 32, 128, 128)   # fp32: SIMT
    assert f(1, 8192, 32, 128, 128, 1, 1, BWD_TENSOR) == 0                          # not covered
    assert f(1, 100, 2, 128, 64, 1, 0, BWD_AUTO) == bwd_ws(2 + 1, 2, 128, 64)      # dv = 64: SIMT
    assert f(1, 100, 2, 128, 64, 1, 0, BWD_TENSOR) == 0
    assert f(2, 0, 2, 128, 128, 2, 0, BWD_AUTO) == 0                                # no tokens
    # the dtype-free query covers either schedule
    for args in [(1, 8192, 32, 128, 128, 1), (3, 100, 2, 64, 64, 3), (1, 100, 2, 128, 64, 1)]:
        for dtype in (0, 1):
            assert lib.kda_chunk_backward_workspace_size(*args) >= f(*args, dtype, BWD_AUTO)


def test_backward_ex_rejects(lib):
    def call(entry, algo, dtype=0, dk=128, dv=128, wsb=1 << 30):
        return entry(A[0], A[1], A[2], A[3], A[4], A[5], A[6], A[7], A[8], A[9], A[10], A[11], A[11] + 0x8000,
                     A[11] + 0x4000, None, 1, 128, 2, dk, dv, 1, dtype, 64, A[0] + 0x8000, wsb, None, algo)
    for entry in (lib.kda_chunk_backward_ex, lib.kda_gdn_chunk_backward_ex):
        assert call(entry, 7) == INVALID                           # no such schedule
        assert call(entry, BWD_TENSOR, dtype=1) == UNSUPPORTED      # fp32 inputs: SIMT only
        assert call(entry, BWD_TENSOR, dk=64, dv=64) == UNSUPPORTED
        assert call(entry, BWD_TENSOR, wsb=2 * 3 * UNIT128 - 16) == WORKSPACE   # one byte row short
        assert lib.kda_last_error().decode() != ""


def backward(lib, **over):
    a = dict(q=A[0], k=A[1], v=A[2], g=A[3], b=A[4], s0=A[5], do=A[6], dF=A[7], dq=A[8], dk_=A[9], dv_=A[10],
             dg=A[11], db=A[11] + 0x8000, ds0=A[11] + 0x4000, cu=None, B=1, T=128, H=2, dk=128, dv=128, N=1,
             dtype=0, chunk=64, ws=A[0] + 0x8000, wsb=1 << 30, st=None)
    a.update(over)
    return lib.kda_chunk_backward(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["do"], a["dF"], a["dq"],
                                  a["dk_"], a["dv_"], a["dg"], a["db"], a["ds0"], a["cu"], a["B"], a["T"], a["H"],
                                  a["dk"], a["dv"], a["N"], a["dtype"], a["chunk"], a["ws"], a["wsb"], a["st"])


@pytest.mark.parametrize("over,code", [
    (dict(do=None), INVALID),
    (dict(dq=None), INVALID),
    (dict(db=None), INVALID),
    (dict(N=2), INVALID),
    (dict(dk=96), UNSUPPORTED),
    (dict(chunk=32), UNSUPPORTED),
    (dict(dtype=5), UNSUPPORTED),
    (dict(do=A[6] + 8), MISALIGNED),
    (dict(dg=A[11] + 4), MISALIGNED),
    (dict(ds0=A[11] + 0x4000 + 8), MISALIGNED),
    (dict(db=A[11] + 0x8000 + 2), MISALIGNED),
    (dict(ws=None, wsb=0), WORKSPACE),
    (dict(wsb=1000), WORKSPACE),
])
def test_backward_rejects(lib, over, code):
    assert backward(lib, **over) == code
    assert lib.kda_last_error().decode() != ""


def test_prologue_entry_points_reject(lib):
    pro = lambda **o: lib.kda_chunk_forward_prologue(
        o.get("q", A[0]), A[1], A[2], o.get("x", A[3]), A[4], A[5], A[6], A[7], None, 1, 128, 2, 128, 128, 1,
        o.get("dtype", 0), 64, o.get("algo", 0), o.get("ws", A[8]), o.get("wsb", 1 << 24), None)
    assert pro(x=None) == INVALID                  # gate pre-activation missing
    assert pro(x=A[3] + 8) == MISALIGNED           # gate below 16-byte alignment
    assert pro(algo=1) == UNSUPPORTED              # the fused schedule takes prepared inputs only
    assert pro(algo=9) == INVALID
    assert pro(ws=None, wsb=0) == WORKSPACE        # two-pass workspace missing
    assert pro(dtype=4) == UNSUPPORTED
    step = lambda **o: lib.kda_recurrent_step_prologue(A[0], A[1], A[2], o.get("x", A[3]), A[4], A[5], A[6], 4, 2,
                                                       128, 128, 0, None)
    assert step(x=None) == INVALID
    assert step(x=A[3] + 4) == MISALIGNED


def test_wait_timeout_hook_rejects_limits(lib):
    assert lib.kda_debug_wait_timeout(0, None) == INVALID
    assert lib.kda_debug_wait_timeout(3_000_000_000, None) == INVALID
