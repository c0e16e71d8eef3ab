"""Host-side checks of the C ABI: the library loads, exports every function that
include/*.h declares, and rejects bad arguments before touching the GPU."""

import ctypes
import glob
import os
import re

import pytest

from mlstm_chunkwise_attention_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for header in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(header).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(?:int|size_t|const\s+char\s*\*|void)\s*\**\s*(mlstm_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from mlstm_chunkwise_attention_b200 import _build
        _build.build()
    return B.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mlstm_fwd", "mlstm_bwd", "mlstm_saved_size", "mlstm_fwd_workspace_size",
                     "mlstm_bwd_workspace_size", "mlstm_status_string", "mlstm_saved_layout"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(B.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in include/ but not exported"


def test_binding_covers_every_declared_symbol():
    assert declared_functions() <= set(B.EXPORTS)


SIZES = dict(B=2, NH=3, T=300, d_qk=128, d_hv=128, chunk=128, variant=B.EXP, dtype=B.BF16)


def sizes(**kw):
    d = dict(SIZES)
    d.update(kw)
    return (d["B"], d["NH"], d["T"], d["d_qk"], d["d_hv"], d["chunk"], d["variant"], d["dtype"])


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(T=-5), 1), (dict(variant=2), 1), (dict(dtype=7), 1),
    (dict(d_qk=0), 1), (dict(chunk=0), 1),
    (dict(d_qk=96), 2), (dict(d_hv=32), 2), (dict(d_qk=512), 2), (dict(chunk=100), 2),
    (dict(chunk=32), 2), (dict(chunk=8192), 2), (dict(B=1 << 16, NH=1 << 10, T=4096), 2),
])
def test_size_validation(lib, kw, status):
    lay = B.SavedLayout()
    assert lib.mlstm_saved_layout(*sizes(**kw), ctypes.byref(lay)) == status
    assert lib.mlstm_saved_size(*sizes(**kw)) == 0
    assert lib.mlstm_bwd_workspace_size(*sizes(**kw)) == 0
    assert lib.mlstm_fwd(None, None, None, None, None, None, None, None, 0, *sizes(**kw), None) == status


def test_null_and_misaligned_pointers_rejected_before_launch(lib):
    fake = 1 << 20  # never dereferenced: validation fails before any launch
    good = [fake] * 6
    assert lib.mlstm_fwd(None, *good[1:], None, None, 0, *sizes(), None) == 1
    assert lib.mlstm_fwd(fake + 4, *good[1:], fake, None, 0, *sizes(), None) == 1
    # no saved buffer and no workspace
    assert lib.mlstm_fwd(*good, None, None, 0, *sizes(), None) == 3
    need = lib.mlstm_fwd_workspace_size(*sizes())
    assert lib.mlstm_fwd(*good, None, fake, need - 1, *sizes(), None) == 3
    bw = lib.mlstm_bwd_workspace_size(*sizes())
    args13 = [fake] * 13
    assert lib.mlstm_bwd(*args13, fake, bw - 1, *sizes(), None) == 3
    assert lib.mlstm_bwd(*args13[:7], None, *args13[8:], fake, bw, *sizes(), None) == 1


def test_empty_problem_is_a_noop(lib):
    for kw in (dict(B=0), dict(NH=0), dict(T=0)):
        assert lib.mlstm_fwd(None, None, None, None, None, None, None, None, 0, *sizes(**kw), None) == 0
        assert lib.mlstm_bwd(*([None] * 13), None, 0, *sizes(**kw), None) == 0
        assert lib.mlstm_fwd_launch_count(*sizes(**kw)) == 0


@pytest.mark.parametrize("L", [128, 512])
def test_saved_layout_regions(lib, L):
    for variant in (B.SIG, B.EXP):
        for dtype in (B.BF16, B.FP32):
            Bn, NH, T, dqk, dhv = 2, 3, 300, 128, 256
            lay = B.mlstm_saved_layout(Bn, NH, T, dqk, dhv, L, variant, dtype)
            NC = (T + L - 1) // L
            tok = Bn * NH * T
            assert lay["gate_b_bytes"] == 4 * tok and lay["gate_li_bytes"] == 4 * tok
            assert lay["gate_m_bytes"] == (4 * tok if variant == B.EXP else 0)
            assert lay["norm_bytes"] == (4 * tok if variant == B.EXP else 0)
            # bf16: hi and lo bf16 planes; fp32: one fp32 plane
            assert lay["state_c_bytes"] == Bn * NH * NC * dqk * dhv * 4
            assert lay["state_n_bytes"] == (Bn * NH * NC * dqk * 4 if variant == B.EXP else 0)
            # per-chunk gate tables of the large-chunk bf16 output kernel:
            # 5 L floats + max(32, L / 32) block maxima per chunk
            xl = dtype == B.BF16 and L >= 256
            assert lay["tile_table_bytes"] == (Bn * NH * NC * (5 * L + max(32, L // 32)) * 4
                                               if xl else 0)
            regions = sorted((lay[n], lay[n + "_bytes"]) for n in
                             ("gate_b", "gate_li", "gate_m", "norm", "state_c", "state_n",
                              "tile_table"))
            end = 0
            for off, nb in regions:
                assert off % 256 == 0 and off >= end
                end = off + nb
            assert lay["total"] >= end
            assert B.mlstm_saved_size(Bn, NH, T, dqk, dhv, L, variant, dtype) == lay["total"]
            assert lib.mlstm_fwd_launch_count(Bn, NH, T, dqk, dhv, L, variant, dtype) > 0
            assert lib.mlstm_bwd_launch_count(Bn, NH, T, dqk, dhv, L, variant, dtype) > 0


def test_status_strings(lib):
    for code in range(6):
        assert B.mlstm_status_string(code)
    assert B.mlstm_status_string(99) == "unknown status"


def test_state_layout_and_argument_errors(lib):
    """Recurrent-state entry points: sizes, and argument errors returned before any launch."""
    for variant in (B.SIG, B.EXP):
        nb = lib.mlstm_state_size(2, 3, 128, 64, variant)
        c = 2 * 3 * 128 * 64 * 4
        if variant == B.SIG:
            assert nb == c
        else:  # C, then n and m on 256-byte boundaries
            n_off = (c + 255) // 256 * 256
            m_off = (n_off + 6 * 128 * 4 + 255) // 256 * 256
            assert nb == (m_off + 6 * 4 + 255) // 256 * 256
    assert lib.mlstm_state_size(2, 3, 100, 64, B.EXP) == 0  # unsupported d_qk
    fake, other = 0x10000, 0x20000  # aligned addresses, never dereferenced
    nb = lib.mlstm_state_size(1, 2, 64, 64, B.EXP)
    args = (fake, fake, fake, fake, fake, fake)
    # overlapping state_in / state_out
    assert lib.mlstm_step(*args, fake, fake + 256, 1, 2, 64, 64, B.EXP, B.BF16, None) == B.STATUS_INVALID
    assert nb > 256
    # NULL state
    assert lib.mlstm_step(*args, None, other, 1, 2, 64, 64, B.EXP, B.BF16, None) == B.STATUS_INVALID
    # misaligned
    assert lib.mlstm_state_zero(fake + 4, 1, 2, 64, 64, B.EXP, None) == B.STATUS_INVALID
    # empty problems are no-ops
    assert lib.mlstm_state_zero(None, 0, 2, 64, 64, B.EXP, None) == 0
    assert lib.mlstm_step(*[None] * 8, 0, 2, 64, 64, B.SIG, B.BF16, None) == 0
    assert lib.mlstm_final_state(None, None, None, None, 0, 2, 5, 64, 64, 64, B.SIG, B.BF16, None) == 0


def test_chunkwise_state_entry_points_argument_errors(lib):
    """mlstm_fwd_state / mlstm_bwd_state: argument errors are returned before any launch."""
    fake, other = 0x10000, 0x20000  # aligned addresses, never dereferenced
    sizes = (1, 2, 256, 64, 64, 64, B.EXP, B.BF16)
    fwd_in = (fake,) * 6 + (fake, None, 0)  # q k v ig fg h, saved, workspace, bytes
    # overlapping initial and final states
    assert lib.mlstm_fwd_state(*fwd_in, fake, fake + 256, *sizes, None) == B.STATUS_INVALID
    # misaligned states
    assert lib.mlstm_fwd_state(*fwd_in, fake + 8, other, *sizes, None) == B.STATUS_INVALID
    assert lib.mlstm_fwd_state(*fwd_in, fake, other + 4, *sizes, None) == B.STATUS_INVALID
    # unsupported sizes come first
    assert lib.mlstm_fwd_state(*fwd_in, fake, other, 1, 2, 256, 100, 64, 64, B.EXP, B.BF16,
                               None) == B.STATUS_UNSUPPORTED
    bwd_in = (fake,) * 8  # q k v ig fg h dh saved
    outs = (fake,) * 5 + (fake, 1 << 30)  # dq dk dv dig dfg, workspace, bytes
    assert lib.mlstm_bwd_state(*bwd_in, fake, fake + 512, None, *outs, *sizes, None) == B.STATUS_INVALID
    assert lib.mlstm_bwd_state(*bwd_in, fake, other + 4, None, *outs, *sizes, None) == B.STATUS_INVALID
    assert lib.mlstm_bwd_state(*bwd_in, fake, other, other + 256, *outs, *sizes, None) == B.STATUS_INVALID
    # empty problems are no-ops
    assert lib.mlstm_fwd_state(*[None] * 8, 0, None, None, 0, 2, 256, 64, 64, 64, B.SIG, B.BF16,
                               None) == 0
    assert lib.mlstm_bwd_state(*[None] * 17, 0, 0, 2, 256, 64, 64, 64, B.SIG, B.BF16, None) == 0


def test_segment_entry_points_argument_errors(lib):
    """mlstm_log_decay / mlstm_state_chain: argument errors before any launch."""
    fake, other, third = 0x10000, 0x40000, 0x80000  # aligned, never dereferenced
    assert lib.mlstm_log_decay(fake, None, 1, 2, 100, B.BF16, None) == B.STATUS_INVALID
    assert lib.mlstm_log_decay(fake + 2, other, 1, 2, 100, B.BF16, None) == B.STATUS_INVALID
    assert lib.mlstm_log_decay(fake, other, 1, 2, 100, 7, None) == B.STATUS_INVALID
    assert lib.mlstm_log_decay(None, None, 0, 2, 100, B.BF16, None) == 0
    # the output must not overlap either input
    assert lib.mlstm_state_chain(fake, other, third, fake + 256, 1, 2, 64, 64, B.EXP, None) == B.STATUS_INVALID
    assert lib.mlstm_state_chain(fake, other, third, other, 1, 2, 64, 64, B.SIG, None) == B.STATUS_INVALID
    assert lib.mlstm_state_chain(fake, other, None, third, 1, 2, 64, 64, B.SIG, None) == B.STATUS_INVALID
    assert lib.mlstm_state_chain(fake, other, third, third + 4, 1, 2, 64, 64, B.SIG, None) == B.STATUS_INVALID
    assert lib.mlstm_state_chain(fake, other, third, 0x100000, 1, 2, 100, 64, B.SIG, None) == B.STATUS_UNSUPPORTED


def test_backward_chain_argument_errors(lib):
    """mlstm_dstate_chain and the state-gradient-only pass: argument errors before any launch."""
    a, b, c, d, g, o = (0x10000 * (i + 1) for i in range(6))  # aligned, never dereferenced
    sz = (1, 2, 64, 64, B.EXP, None)
    assert lib.mlstm_dstate_chain(a, b, c, d, None, o, *sz) == B.STATUS_INVALID
    assert lib.mlstm_dstate_chain(a, b, c, d, g, a + 256, *sz) == B.STATUS_INVALID  # overlaps dstate_local
    assert lib.mlstm_dstate_chain(a, b, c, d, g, b, *sz) == B.STATUS_INVALID        # overlaps dstate_out
    assert lib.mlstm_dstate_chain(a, b, c, d, g, o + 8, *sz) == B.STATUS_INVALID
    assert lib.mlstm_dstate_chain(None, None, None, None, None, None, 0, 2, 64, 64, B.EXP, None) == 0
    # state-gradient-only pass: all five gradient outputs NULL needs a dstate_in
    sizes = (1, 2, 256, 64, 64, 64, B.SIG, B.BF16)
    ins = (a,) * 8
    assert lib.mlstm_bwd_state(*ins, None, None, None, None, None, None, None, None, b, 1 << 30,
                               *sizes, None) == B.STATUS_INVALID
    # some but not all of the five outputs
    assert lib.mlstm_bwd_state(*ins, None, c, None, d, None, None, None, None, b, 1 << 30,
                               *sizes, None) == B.STATUS_INVALID


def _plan(pass_, sizes):
    n = (B.mlstm_fwd_launch_count if pass_ == 0 else B.mlstm_bwd_launch_count)(*sizes)
    return [B.mlstm_launch_name(pass_, i, *sizes) for i in range(n)]


@pytest.mark.parametrize("variant", [B.SIG, B.EXP], ids=["sig", "exp"])
def test_launch_plans_choose_the_walkers_on_their_shape(lib, variant):
    """bf16, chunk 128, d_qk = d_hv = 128: the forward walker replaces the state and output
    kernels, the backward walker the state-gradient, dk and dv kernels (dq stays); any other
    chunk, head dim or dtype keeps the separate kernels."""
    walk = (2, 4, 1000, 128, 128, 128, variant, B.BF16)
    assert _plan(0, walk) == ["gate_prep", "fwd_walk_tc"]
    assert _plan(1, walk) == ["bwd_token_prep", "dkv_walk_tc", "dq_tc", "gate_grad"]
    for other in [(2, 4, 1000, 128, 128, 256, variant, B.BF16),
                  (2, 4, 1000, 64, 128, 128, variant, B.BF16),
                  (2, 4, 1000, 128, 256, 128, variant, B.BF16),
                  (2, 4, 1000, 128, 128, 128, variant, B.FP32)]:
        names = _plan(0, other) + _plan(1, other)
        assert not any("walk" in n for n in names), (other, names)
        assert any(n.startswith("state_fwd") for n in names) and any(n.startswith("dk_") for n in names)


@pytest.mark.parametrize("variant", [B.SIG, B.EXP], ids=["sig", "exp"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_launch_plans_put_every_bf16_chunk_size_on_tensor_cores(lib, variant, d):
    """bf16 runs every chunk size on tcgen05 kernels: chunk 64 and 128 on the one-tile
    output kernel (or the walkers), chunk >= 256 on the large-chunk kernel, the backward on
    the tensor-core state-gradient and dq / dk / dv kernels.  fp32 I/O keeps the CUDA-core
    kernels (a bf16 operand cannot meet its 1e-4 bar)."""
    for L in (64, 128, 256, 1024):
        sizes = (2, 4, 2048, d, d, L, variant, B.BF16)
        names = _plan(0, sizes) + _plan(1, sizes)
        assert not any(n.endswith("_simt") for n in names), (L, names)
        fwd_out = _plan(0, sizes)[-1]
        if L <= 128:
            assert fwd_out in ("output_fwd_tc", "fwd_walk_tc"), (L, fwd_out)
        else:
            assert fwd_out == "output_fwd_xl", (L, fwd_out)
    names = _plan(0, (2, 4, 2048, d, d, 64, variant, B.FP32)) + _plan(1, (2, 4, 2048, d, d, 64, variant, B.FP32))
    assert all(n.endswith("_simt") for n in names if n not in ("gate_prep", "bwd_token_prep", "gate_grad"))


@pytest.mark.parametrize("variant", [B.SIG, B.EXP], ids=["sig", "exp"])
def test_launch_plans_large_chunk_backward(lib, variant):
    """bf16, d_qk = d_hv = 128, chunk >= 256: the backward's intra-chunk products run on the
    large-chunk kernels after their gate table; other head dims keep the one-tile kernels."""
    for L in (256, 512, 1024, 4096):
        assert _plan(1, (8, 32, 5000, 128, 128, L, variant, B.BF16)) == [
            "bwd_token_prep", "state_bwd_tc", "bwd_xl_table", "dq_xl", "dk_xl", "dv_xl", "gate_grad"]
    for other in [(2, 4, 5000, 64, 64, 256, variant, B.BF16),
                  (2, 4, 5000, 128, 256, 512, variant, B.BF16),
                  (2, 4, 5000, 128, 128, 128, variant, B.BF16),
                  (2, 4, 5000, 128, 128, 256, variant, B.FP32)]:
        assert not any(n.endswith("_xl") and n != "output_fwd_xl" for n in _plan(1, other)), other


@pytest.mark.parametrize("variant", [B.SIG, B.EXP], ids=["sig", "exp"])
def test_launch_plans_split_state_walks_for_few_heads(lib, variant):
    """Few heads with many chunks: the state kernels walk each head's chunks in segments and a
    completion pass follows each; enough heads to fill the GPU, or fewer than eight chunks
    (at least four per segment), keep one walk per head."""
    long_few = (1, 8, 65536, 256, 512, 1024, variant, B.BF16)  # the long-context workload
    fwd, bwd = _plan(0, long_few), _plan(1, long_few)
    assert fwd[fwd.index("state_fwd_tc") + 1] == "state_fwd_fix", fwd
    assert bwd[bwd.index("state_bwd_tc") + 1] == "state_bwd_fix", bwd
    assert len(bwd) <= 10  # the plan's step array holds ten
    # the gate gradients too run over segments of the sequence, after their totals
    assert bwd[-2:] == ["gate_grad_sums", "gate_grad"], bwd
    assert _plan(1, (8, 32, 8192, 128, 128, 128, variant, B.BF16))[-1] == "gate_grad"
    assert "gate_grad_sums" not in _plan(1, (8, 32, 8192, 128, 128, 128, variant, B.BF16))
    walk_few = _plan(1, (1, 4, 32768, 128, 128, 128, variant, B.BF16))
    assert walk_few[-2:] == ["gate_grad_sums", "gate_grad"], walk_few
    for sizes in [(8, 32, 8192, 128, 128, 256, variant, B.BF16),   # 256 heads: one walk each
                  (1, 2, 448, 64, 64, 64, variant, B.BF16)]:       # 7 chunks: too few to split
        names = _plan(0, sizes) + _plan(1, sizes)
        assert not any(n.endswith("_fix") for n in names), (sizes, names)
    assert "state_bwd_fix" in _plan(1, (1, 2, 4096, 128, 128, 256, variant, B.BF16))


def test_serial_launch_switch_needs_no_device(lib):
    """mlstm_set_serial_launches only sets a per-thread flag: no CUDA call, always MLSTM_OK."""
    assert lib.mlstm_set_serial_launches(1) == 0
    assert lib.mlstm_set_serial_launches(0) == 0
    assert lib.mlstm_set_serial_launches(7) == 0
    assert lib.mlstm_set_serial_launches(0) == 0


def test_bench_accounts_for_every_planned_kernel(lib):
    """Every kernel a launch plan can name has an algorithmic (FLOPs, bytes) entry and a source
    file in bench.py, so the bench's per-kernel roofline never meets an unknown kernel."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    seen = set()
    for dt in (B.BF16, B.FP32):
        for var in (B.SIG, B.EXP):
            for (Bn, NH, T, dqk, dhv) in [(2, 4, 1000, 128, 128), (1, 2, 300, 64, 64),
                                         (1, 8, 65536, 256, 512), (8, 32, 4096, 128, 128),
                                         (1, 4, 32768, 128, 128), (2, 2, 640, 256, 256)]:
                for L in (64, 128, 256, 512, 1024):
                    sizes = (Bn, NH, T, dqk, dhv, L, var, dt)
                    names = _plan(0, sizes) + _plan(1, sizes)
                    costs = bench.kernel_costs(T, dqk, dhv, L, var == B.EXP, 2 if dt == B.BF16 else 4)
                    for n in names:
                        assert n in costs, (sizes, n)
                        assert n in bench.KERNEL_SOURCES, (sizes, n)
                        assert bench.kernel_bound(n) in ("hbm", "tensor", "alu")
                        assert os.path.exists(os.path.join(ROOT, "mlstm_chunkwise_attention_b200",
                                                           "csrc", bench.KERNEL_SOURCES[n]))
                    seen.update(names)
    # the walkers, the large-chunk kernels, the segmented walks and the CUDA-core path all occur
    for n in ("fwd_walk_tc", "dkv_walk_tc", "output_fwd_xl", "dq_xl", "state_fwd_fix",
              "gate_grad_sums", "output_fwd_simt", "dq_simt"):
        assert n in seen, n
