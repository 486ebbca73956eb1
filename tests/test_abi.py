"""The C-ABI library: it loads, exports every entry point include/gdn2.h
declares, and rejects bad arguments on the host before anything is launched
(these calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_gdn2_b200 as g
from gated_delta_rule_gdn2_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "gdn2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn2_\w+)\s*\(", text)))


def test_build_is_current():
    assert gbuild.build() == g.LIB_PATH
    assert os.path.exists(g.LIB_PATH)


def test_exports_every_declared_symbol():
    lib = ctypes.CDLL(g.LIB_PATH)
    syms = declared_symbols()
    assert len(syms) >= 8
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(g.binding.SIGNATURES)


def test_version_and_status_strings():
    assert g.gdn2_version() == 100
    for code, name in g.STATUS.items():
        assert g.gdn2_status_string(code).startswith(name)
    assert "unknown" in g.gdn2_status_string(-99)


def _fwd(**kw):
    a = dict(q=16, k=16, v=16, log_alpha=16, b=16, w=16, S0=None, o=16, S_T=None, B=1, T=64, H=1,
             dk=64, dv=64, dtype=g.GDN2_BF16, ws=16, ws_bytes=1 << 30, stream=0)
    a.update(kw)
    return g.gdn2_chunk_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["b"], a["w"], a["S0"], a["o"],
                            a["S_T"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["dtype"], a["ws"],
                            a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(dk=96), -2), (dict(dv=32), -2), (dict(dtype=7), -2),
    (dict(B=-1), -1), (dict(T=-5), -1), (dict(H=-1), -1),
    (dict(q=None), -1), (dict(o=None), -1), (dict(k=24), -1), (dict(S0=8), -1),
    (dict(ws=None), -5), (dict(ws_bytes=16), -5),
])
def test_chunk_fwd_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def test_empty_batch_is_a_noop():
    assert _fwd(B=0, q=None, k=None, v=None, log_alpha=None, b=None, w=None, o=None) == 0
    assert _fwd(H=0, q=None, k=None, v=None, log_alpha=None, b=None, w=None, o=None) == 0


def test_decode_and_bwd_reject_bad_arguments():
    assert g.gdn2_decode_step(16, 16, 16, 16, 16, 16, None, 16, 1, 1, 64, 64, 0, 0) == -1
    assert g.gdn2_decode_step(16, 16, 16, 16, 16, 16, 16, 16, 1, 1, 64, 80, 0, 0) == -2
    assert g.gdn2_decode_step(16, 16, 16, 16, 16, 16, 20, 16, 1, 1, 64, 64, 0, 0) == -1
    args = [16] * 6 + [None, 16, None] + [16] * 6 + [None]
    assert g.gdn2_chunk_bwd(*args, 1, 64, 1, 64, 64, 0, None, 0, 0) == -5
    args[7] = None  # dO
    assert g.gdn2_chunk_bwd(*args, 1, 64, 1, 64, 64, 0, 16, 1 << 40, 0) == -1
    assert g.gdn2_chunk_bwd(*([16] * 16), 1, 64, 1, 128, 64, 3, 16, 1 << 40, 0) == -2


def test_workspace_sizes():
    assert g.gdn2_chunk_fwd_workspace(8, 4096, 16, 128, 128, g.GDN2_BF16) == 8 * 16 * 64 * 128 * 4
    # few long sequences: the segmented forward's workspace (P = 5 segments of
    # B1 H16 T32768 on 148 SMs, 16 * (2 * 5 - 1) = 144 CTAs: their per-CTA
    # scratch, the bf16 rows Phi_t^T q_t like the token tensor, and the fp32
    # [128][128] end states of 5 segments, transitions and start states of 4)
    r = lambda x: (x + 255) // 256 * 256
    seg = (r(144 * 64 * 128 * 4) + r(32768 * 16 * 128 * 2) + r(5 * 16 * 128 * 128 * 4)
           + 2 * r(4 * 16 * 128 * 128 * 4))
    # ... and, for the saving forward of segmented training, the start states
    # of the 5 segments, their offsets and the packed forward's scratch
    train = seg + r(5 * 16 * 128 * 128 * 4) + r(6 * 4) + r(5 * 16 * 64 * 128 * 4)
    assert g.gdn2_chunk_fwd_workspace(1, 32768, 16, 128, 128, g.GDN2_BF16) == max(seg, train)
    # too short for two segments of 8 chunks: the plain size
    assert g.gdn2_chunk_fwd_workspace(1, 960, 16, 128, 128, g.GDN2_BF16) == 16 * 64 * 128 * 4
    # too many sequences to split (3 * 64 CTAs > 148): the plain size
    assert g.gdn2_chunk_fwd_workspace(4, 32768, 16, 128, 128, g.GDN2_BF16) == 4 * 16 * 64 * 128 * 4
    # a ragged length never splits
    assert g.gdn2_chunk_fwd_workspace(1, 32767, 16, 128, 128, g.GDN2_BF16) == 16 * 64 * 128 * 4
    assert g.gdn2_chunk_fwd_workspace(8, 4096, 16, 128, 128, g.GDN2_FP32) == 0
    assert g.gdn2_chunk_fwd_workspace(0, 4096, 16, 128, 128, g.GDN2_BF16) == 0
    assert g.gdn2_chunk_bwd_workspace(8, 4096, 16, 128, 128, g.GDN2_BF16) > 0
    assert g.gdn2_chunk_bwd_workspace(8, 4096, 16, 96, 128, g.GDN2_BF16) == 0


def test_saved_state_entry_points_validate():
    B, T, H = 2, 100, 3
    n = g.gdn2_chunk_states_bytes(B, T, H, 128, 128, g.GDN2_BF16)
    # ceil(100/64) + 1 bf16 chunk-boundary states, then per chunk the bf16
    # tiles T, M (64 x 64) and U (64 x dv), then (dk = dv = 128 only) per chunk
    # the decayed operands Qt, Gt, Kb (64 x 128 each); every region is a
    # multiple of 256 bytes here
    assert n == B * H * (2 + 1) * 128 * 128 * 2 + B * H * 2 * (2 * 64 * 64 + 64 * 128) * 2 + \
        B * H * 2 * 3 * 64 * 128 * 2
    assert g.gdn2_chunk_states_bytes(B, T, H, 64, 64, g.GDN2_BF16) == \
        B * H * (2 + 1) * 64 * 64 * 2 + B * H * 2 * (2 * 64 * 64 + 64 * 64) * 2
    assert g.gdn2_chunk_states_bytes(B, T, H, 128, 128, g.GDN2_FP32) == 0
    assert 0 < g.gdn2_chunk_bwd_saved_workspace(B, T, H, 128, 128, g.GDN2_BF16) < \
        g.gdn2_chunk_bwd_workspace(B, T, H, 128, 128, g.GDN2_BF16)
    # missing or misaligned state buffer is refused before any launch
    args = [16] * 6 + [None, 16, None, None] + [16] * 6 + [None]
    assert g.gdn2_chunk_bwd_saved(*args, B, T, H, 128, 128, 0, 16, 1 << 40, 0) == -1
    args[9] = 24
    assert g.gdn2_chunk_bwd_saved(*args, B, T, H, 128, 128, 0, 16, 1 << 40, 0) == -1
    assert g.gdn2_chunk_fwd_save(16, 16, 16, 16, 16, 16, None, 16, None, None, B, T, H, 128, 128, 0, 16,
                                 1 << 40, 0) == -1


def test_varlen_rejects_missing_or_misaligned_offsets():
    args = [16] * 6 + [None, 16, None]
    assert g.gdn2_chunk_fwd_varlen(*args, None, 2, 100, 1, 128, 128, g.GDN2_BF16, 16, 1 << 30, 0) == -1
    assert g.gdn2_chunk_fwd_varlen(*args, 18, 2, 100, 1, 128, 128, g.GDN2_BF16, 16, 1 << 30, 0) == -1
    assert g.gdn2_chunk_fwd_varlen(*args, 16, 2, 100, 1, 96, 128, g.GDN2_BF16, 16, 1 << 30, 0) == -2
    assert g.gdn2_chunk_fwd_varlen(*args, 16, 2, 100, 1, 128, 128, g.GDN2_BF16, 16, 0, 0) == -5
    # N = 0 is a no-op; total_T = 0 only copies the states (none here)
    assert g.gdn2_chunk_fwd_varlen(*args, 16, 0, 100, 1, 128, 128, g.GDN2_BF16, None, 0, 0) == 0
    assert g.gdn2_chunk_fwd_varlen(*args, 16, 2, 0, 1, 128, 128, g.GDN2_BF16, None, 0, 0) == 0
    gargs = [16] * 6 + [None, 16, None] + [16] * 6 + [None]
    assert g.gdn2_chunk_bwd_varlen(*gargs, None, 2, 100, 1, 128, 128, g.GDN2_BF16, 16, 1 << 40, 0) == -1
    assert g.gdn2_chunk_bwd_varlen(*gargs, 16, 2, 100, 1, 128, 128, g.GDN2_BF16, 16, 16, 0) == -5


def test_varlen_buffer_sizes_depend_on_totals_only():
    # the saved-state buffer of a packed batch: per head floor(T/64) + 2N
    # state slots and floor(T/64) + N chunk slots, whatever the lengths
    N, T, H = 5, 1000, 2
    st = g.gdn2_chunk_states_varlen_bytes(N, T, H, 128, 128, g.GDN2_BF16)
    states = H * (T // 64 + 2 * N) * 128 * 128 * 2
    chunks = H * (T // 64 + N)
    intra = chunks * (2 * 64 * 64 * 2 + 64 * 128 * 2)
    ops = chunks * 3 * 64 * 128 * 2
    r = lambda x: (x + 255) // 256 * 256
    assert st == r(states) + r(intra) + ops
    assert g.gdn2_chunk_fwd_varlen_workspace(N, T, H, 128, 128, g.GDN2_BF16) == N * H * 64 * 128 * 4
    assert g.gdn2_chunk_states_varlen_bytes(N, T, H, 128, 128, g.GDN2_FP32) == 0


def test_reduced_gate_entry_points_validate():
    """KDA / Gated DeltaNet calls: a missing or misaligned scalar gate, a missing
    gradient and unsupported sizes are refused on the host."""
    P = 16  # a 16-byte aligned stand-in address (never dereferenced: the calls fail first)
    fwd = lambda **kw: g.gdn2_chunk_fwd_kda(*[kw.get(n, P) for n in ("q", "k", "v", "la", "beta")], None,
                                            kw.get("o", P), None, 1, 64, 1, kw.get("dk", 128), 128,
                                            g.GDN2_BF16, P, 1 << 30, 0)
    assert fwd(beta=None) == -1
    assert fwd(beta=17) == -1          # not even element-aligned for bf16
    assert fwd(dk=96) == -2
    assert g.gdn2_chunk_fwd_gdn(P, P, P, 17, P, None, P, None, 1, 64, 1, 128, 128, g.GDN2_BF16, P, 1 << 30, 0) == -1
    assert g.gdn2_chunk_fwd_gdn(P, P, P, P, P, None, P, None, 0, 64, 1, 128, 128, g.GDN2_BF16, None, 0, 0) == 0
    bwd = [P] * 5 + [None, P, None] + [P] * 4
    assert g.gdn2_chunk_bwd_kda(*bwd, None, None, 1, 64, 1, 128, 128, g.GDN2_BF16, P, 1 << 40, 0) == -1  # no dbeta
    assert g.gdn2_chunk_bwd_gdn(*bwd, P, None, 1, 64, 1, 96, 128, g.GDN2_BF16, P, 1 << 40, 0) == -2
    assert g.gdn2_decode_step_kda(P, P, P, P, None, P, P, 1, 1, 128, 128, g.GDN2_BF16, 0) == -1
    assert g.gdn2_decode_step_gdn(P, P, P, 19, P, P, P, 1, 1, 128, 128, g.GDN2_BF16, 0) == -1


def test_gated_forward_and_layer_entry_points_validate():
    P = 16
    toks = [P] * 6
    # the fused output gate needs g and gamma
    assert g.gdn2_chunk_fwd_gated(*toks, None, None, P, P, None, 1, 64, 1, 128, 128, g.GDN2_BF16, P, 1 << 30, 0) == -1
    assert g.gdn2_chunk_fwd_gated(*toks, None, P, None, P, None, 1, 64, 1, 128, 128, g.GDN2_BF16, P, 1 << 30, 0) == -1
    # prologue: filter width 1..4, head sizes 64 / 128, 16-byte pointers; no tokens = no-op
    pro = lambda K=4, B=1, T=64, dk=128, xq=P: g.gdn2_prologue_fwd(xq, P, P, P, P, P, K, P, P, P, P, P, P, P, P, P,
                                                                  None, B, T, 2, dk, 128, g.GDN2_BF16, 0)
    assert pro(K=0) == -2 and pro(K=5) == -2 and pro(dk=96) == -2
    assert pro(B=-1) == -1 and pro(xq=24) == -1
    assert pro(T=0) == 0 and pro(B=0) == 0
    # its backward's workspace: one fp32 partial per 64-row block, head, filter tap and channel
    assert g.gdn2_prologue_bwd_workspace(2, 100, 3, 128, 64, 4, 0) == 4 * 3 * (2 * 128 + 64) * 4 * 4
    assert g.gdn2_prologue_bwd_workspace(2, 100, 3, 128, 64, 4, 1) == 2 * 3 * (2 * 128 + 64) * 4 * 4
    assert g.gdn2_prologue_bwd_workspace(2, 100, 3, 128, 64, 5, 0) == 0
    assert g.gdn2_prologue_bwd(*[P] * 6, 4, *[P] * 18, None, 1, 64, 2, 128, 128, g.GDN2_BF16, P, 16, 0) == -5
    # output gate: rows >= 0, dv 64 / 128, aligned pointers, enough workspace
    assert g.gdn2_output_gate_fwd(P, P, P, P, -1, 2, 128, g.GDN2_BF16, 0) == -1
    assert g.gdn2_output_gate_fwd(P, P, P, P, 64, 2, 96, g.GDN2_BF16, 0) == -2
    assert g.gdn2_output_gate_fwd(24, P, P, P, 64, 2, 128, g.GDN2_BF16, 0) == -1
    assert g.gdn2_output_gate_fwd(P, P, P, P, 0, 2, 128, g.GDN2_BF16, 0) == 0
    assert g.gdn2_output_gate_bwd_workspace(100, 3, 128) == 2 * 3 * 128 * 4
    assert g.gdn2_output_gate_bwd(*[P] * 7, 100, 3, 128, g.GDN2_BF16, P, 16, 0) == -5


def test_debug_knobs_reject_out_of_range_values():
    assert g.gdn2_debug_set(7, 0) == -1
    assert g.gdn2_debug_set(g.GDN2_DEBUG_WAIT_LIMIT if hasattr(g, "GDN2_DEBUG_WAIT_LIMIT") else 0, -1) == -1
    assert g.gdn2_debug_set(1, -2) == -1
