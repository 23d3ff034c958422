"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/ringattn.h declares, and rejects bad arguments
before touching the device."""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from exact_blockwise_long_b200 import build
    build.build()
    from exact_blockwise_long_b200 import _lib
    return _lib.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ringattn.h")).read()
    return sorted(set(re.findall(r"RA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = declared_symbols()
    for must in ("ringattn_fwd", "ringattn_bwd", "blockwise_ffn", "ringattn_merge", "ringattn_fwd_step"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    from exact_blockwise_long_b200 import _lib
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_only_declared_symbols_are_exported():
    """Hidden visibility: the dynamic symbol table holds only the ABI."""
    import subprocess
    from exact_blockwise_long_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    ours = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and ("ringattn" in ln or "blockwise" in ln)}
    assert ours == set(declared_symbols())


FAKE = 0x10000  # aligned, never dereferenced: validation fails first
MIS = 0x10001


def fwd(L, q=FAKE, out=FAKE, lse=FAKE, B=1, H=1, N=1024, D=128, dtype=0, S=4, qc=128, kc=128, causal=1):
    return L.ringattn_fwd(q, FAKE, FAKE, out, lse, B, H, N, D, dtype, S, qc, kc, causal, 0.0, None)


def test_fwd_argument_errors(L):
    assert fwd(L, q=None) == -1                     # null pointer
    assert fwd(L, N=-128) == -1                     # negative size
    assert fwd(L, causal=2) == -1
    assert fwd(L, dtype=7) == -3                    # dtype
    assert fwd(L, D=96) == -5                       # head dim not built
    assert fwd(L, N=1000) == -2                     # N % S
    assert fwd(L, N=1024, S=8, qc=256) == -2        # chunk larger than shard
    assert fwd(L, N=1536, S=4, qc=256) == -2        # shard 384 not divisible by 256
    assert fwd(L, qc=64) == -2                      # bf16 tiles are 128
    assert fwd(L, q=MIS) == -4                      # alignment
    assert fwd(L, lse=MIS) == -4
    assert fwd(L, out=None) == -1


def test_fwd_empty_extents_are_noops(L):
    assert fwd(L, B=0, q=None, out=None, lse=None) == 0
    assert fwd(L, N=0, q=None, out=None, lse=None) == 0
    assert fwd(L, H=0) == 0


def test_step_and_merge_argument_errors(L):
    st = L.ringattn_fwd_step
    assert st(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1024, 128, 0, 4, 128, 128, 1, 0.0, 4, None) == -1  # t >= S
    assert st(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1024, 128, 0, 4, 128, 128, 1, 0.0, -1, None) == -1
    assert st(FAKE, FAKE, FAKE, None, FAKE, 1, 1, 1024, 128, 0, 4, 128, 128, 1, 0.0, 0, None) == -1
    m = L.ringattn_merge
    assert m(FAKE, FAKE, FAKE, FAKE, 10, 6, None) == -2     # D % 4
    assert m(None, FAKE, FAKE, FAKE, 10, 8, None) == -1
    assert m(MIS, FAKE, FAKE, FAKE, 10, 8, None) == -4
    assert m(FAKE, FAKE, FAKE, FAKE, 0, 8, None) == 0       # nothing to merge


def test_bwd_workspace_contract(L):
    rows = 32 * 32768
    ws = L.ringattn_bwd_workspace_size(1, 32, 32768, 128)
    # D_i and lse*log2(e) (fp32 rows), then the fused pass's fp32 dQ accumulator
    assert ws == 2 * rows * 4 + rows * 128 * 4
    assert L.ringattn_bwd_workspace_size(1, 32, 32768, 64) == 2 * rows * 4 + rows * 64 * 4
    assert L.ringattn_bwd_workspace_size(0, 1, 1, 1) == 0
    b = L.ringattn_bwd
    ws = L.ringattn_bwd_workspace_size(1, 1, 1024, 128)
    args = [FAKE] * 9 + [1, 1, 1024, 128, 0, 4, 128, 128, 1, 0.0]
    assert b(*args, FAKE, ws - 1, None) == -8          # too small
    assert b(*args, None, ws, None) == -8              # missing
    assert b(*(args[:13] + [1] + args[14:]), FAKE, ws, None) == -5  # fp32 backward not built
    ph = L.ringattn_bwd_phase
    assert ph(*args, FAKE, ws, 0, None) == -1           # empty phase mask
    assert ph(*args, FAKE, ws, 32, None) == -1          # unknown phase bit
    assert ph(*args, FAKE, 2 * 1024 * 4, 8, None) == -8  # the fused pass needs the dQ accumulator
    args64 = args[:12] + [64] + args[13:]
    assert ph(*args64, FAKE, 2 * 1024 * 4, 8, None) == -8  # d = 64 fused pass: the accumulator too


def test_kernel_plan(L):
    """The plan names the kernels a call launches; the shape rules apply."""
    plan = L.ringattn_kernel_plan
    assert plan(0, 1024, 64, 1, 4) == b"fwd_simt_kernel"
    assert plan(1, 32768, 128, 0, 16) == b"bwd_preprocess_kernel+bwd_fused_kernel+bwd_dq_convert_kernel"
    assert plan(1, 8192, 64, 0, 8) == b"bwd_preprocess_kernel+bwd_fused_kernel+bwd_dq_convert_kernel"
    assert plan(1, 1024, 64, 1, 4) is None              # no fp32 backward
    assert plan(0, 1000, 128, 0, 16) is None            # N % S
    assert plan(0, 1024, 96, 0, 4) is None              # D
    assert plan(2, 1024, 128, 0, 4) is None             # op


def test_ffn_contract(L):
    assert L.blockwise_ffn_workspace_size(2048, 11008, 0) == 2048 * 11008 * 2
    f = L.blockwise_ffn
    good = [FAKE] * 5 + [4096, 4096, 11008, 2048, 0]
    ws = L.blockwise_ffn_workspace_size(2048, 11008, 0)
    assert f(*good[:5], 4000, 4096, 11008, 2048, 0, FAKE, ws, None) == -2   # T % chunk
    assert f(*good[:5], 4096, 4096, 11000, 2048, 0, FAKE, ws, None) == -2   # d_ff % 128
    assert f(*good, FAKE, ws - 2, None) == -8
    assert f(*good[:9], 5, FAKE, ws, None) == -3
    assert f(*good[:5], 0, 4096, 11008, 2048, 0, None, 0, None) == 0        # no tokens


def test_status_strings(L):
    for code in range(-8, 1):
        assert L.ringattn_status_string(code)
    assert L.ringattn_version() >= 100


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle and has no CPU fallback."""
    pkg = os.path.join(ROOT, "exact_blockwise_long_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn


def test_ffn_bwd_contract(L):
    f = L.blockwise_ffn_bwd
    ws = L.blockwise_ffn_bwd_workspace_size(2048, 11008, 0)
    assert ws == 2048 * 11008 * (4 + 3 * 2)          # dh fp32 + dg, du, h bf16
    assert L.blockwise_ffn_bwd_workspace_size(2048, 11008, 1) == 0
    ptrs = [FAKE] * 9
    assert f(*ptrs, 4000, 4096, 11008, 2048, 0, FAKE, ws, None) == -2          # T % chunk
    assert f(*ptrs, 4096, 4096, 11000, 2048, 0, FAKE, ws, None) == -2          # d_ff % 128
    assert f(*ptrs, 4096, 4096, 11008, 2048, 1, FAKE, ws, None) == -5          # fp32 not built
    assert f(*ptrs, 4096, 4096, 11008, 2048, 9, FAKE, ws, None) == -3
    assert f(*ptrs, 4096, 4096, 11008, 2048, 0, FAKE, ws - 16, None) == -8
    assert f(*([MIS] + ptrs[1:]), 4096, 4096, 11008, 2048, 0, FAKE, ws, None) == -4
    assert f(*([FAKE] * 6 + [None] + [FAKE] * 2), 4096, 4096, 11008, 2048, 0, FAKE, ws, None) == -1


def test_layer_contract(L):
    B, N, H, D, dff = 1, 4096, 32, 128, 11008
    saved = L.blockwise_layer_saved_size(B, N, H, D)
    dm = H * D
    assert saved >= 7 * N * dm * 2 + 3 * N * 4        # seven bf16 activations, lse and two rstd rows
    fws = L.blockwise_layer_fwd_workspace_size(2048, dff)
    bws = L.blockwise_layer_bwd_workspace_size(B, N, H, D, dff, 2048)
    assert fws == 2048 * dff * 2 and bws > 7 * N * dm * 2
    fwd = L.blockwise_layer_fwd
    p12 = [FAKE] * 12

    def fw(*, ptrs=p12, B=B, N=N, H=H, D=D, dff=dff, S=2, qc=2048, kc=2048, causal=1, fc=2048, eps=1e-5,
           sv=saved, ws=FAKE, wsb=fws):
        return fwd(*ptrs, sv, B, N, H, D, dff, S, qc, kc, causal, fc, eps, ws, wsb, None, None)

    assert fw(S=3) == -2                 # N % S
    assert fw(D=96) == -5                # head dim
    assert fw(H=24) == -5                # d_model 3072 not built (RMS norm rows)
    assert fw(fc=1000) == -2             # ffn chunk
    assert fw(eps=0.0) == -1
    assert fw(sv=saved - 1) == -8
    assert fw(wsb=fws - 1) == -8
    assert fw(ptrs=[None] + p12[1:]) == -1
    assert fw(ptrs=p12[:5] + [MIS] + p12[6:]) == -4
    assert fw(B=0, ptrs=[None] * 12, ws=None, wsb=0) == 0   # no tokens: nothing to do
    bwd = L.blockwise_layer_bwd
    grads = [FAKE] * 9

    def bw(*, B=B, S=2, g=grads, wsb=bws):
        return bwd(*([FAKE] * 11), saved, FAKE, FAKE, *g, B, N, H, D, dff, S, 2048, 2048, 1, 2048, FAKE, wsb,
                   None, None)

    assert bw(S=3) == -2
    assert bw(wsb=bws - 1) == -8
    assert bw(g=[None] + grads[1:]) == -1
    assert bw(B=0, g=[MIS] + grads[1:]) == -4   # no tokens: the gradients must still be valid


def test_accumulate_and_cast_contract(L):
    assert L.ringattn_accumulate(None, FAKE, 16, 0, None) == -1
    assert L.ringattn_accumulate(FAKE, FAKE, -1, 0, None) == -1
    assert L.ringattn_accumulate(FAKE, FAKE, 16, 5, None) == -3
    assert L.ringattn_accumulate(MIS, FAKE, 16, 0, None) == -4
    assert L.ringattn_accumulate(None, None, 0, 0, None) == 0   # nothing to do
    assert L.ringattn_cast(FAKE, None, 16, 0, None) == -1
    assert L.ringattn_cast(FAKE, MIS, 16, 0, None) == -4
    assert L.ringattn_cast(None, None, 0, 1, None) == 0


def test_build_checks_launch_registers():
    """A kernel whose register split needs an exact launch register count
    fails the build when ptxas lands on another count."""
    from exact_blockwise_long_b200 import build
    log = ("ptxas info    : Compiling entry function '_ZN2ra_bwd_fused_kernelILi128EE' for 'sm_100a'\n"
           "ptxas info    : Function properties for _ZN2ra_bwd_fused_kernelILi128EE\n"
           "    0 bytes stack frame, 0 bytes spill stores, 0 bytes spill loads\n"
           "ptxas info    : Used 128 registers, used 1 barriers\n"
           "ptxas info    : Compiling entry function '_ZN2ra_bwd_kv_kernelILi128EE' for 'sm_100a'\n"
           "ptxas info    : Used 161 registers, used 1 barriers\n")
    assert build.kernel_registers(log) == {"_ZN2ra_bwd_fused_kernelILi128EE": 128, "_ZN2ra_bwd_kv_kernelILi128EE": 161}
    build.check_launch_registers("csrc/bwd_tc.cu", log)
    with pytest.raises(RuntimeError, match="exactly 128"):
        build.check_launch_registers("csrc/bwd_tc.cu", log.replace("Used 128", "Used 120"))
    with pytest.raises(RuntimeError, match="no registers"):
        build.check_launch_registers("csrc/fwd_tc.cu", log)


def test_checked_build_exports_the_abi():
    """The bounds-checked build (-DRA_CHECKED) compiles from the same sources
    and exports the same entry points."""
    from exact_blockwise_long_b200 import _lib, build
    h = _lib.load(build.build(checked=True))
    for name in declared_symbols():
        assert hasattr(h, name), name
