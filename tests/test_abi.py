"""The C-ABI library: it loads, exports every function include/moe.h declares,
and rejects bad arguments on the host before launching anything (CPU only)."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

import mixture_experts_layer_62_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:int|int32_t|size_t|long\s+long|const\s+char\s*\*)\s+(moe_\w+)\s*\(", src,
                       flags=re.M)
    assert names, "no declarations parsed"
    return sorted(set(names))


def test_library_loads_and_exports_every_declared_symbol():
    lib = moe.lib
    names = declared_functions()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(moe_\w+)", out))
    assert set(names) <= exported
    # nothing exported under the moe_ prefix that the header does not declare
    assert exported <= set(names), exported - set(names)


def test_wait_limit_is_settable_and_restorable():
    # host-side setting only (nothing launched): the previous value comes back,
    # and a non-positive value restores the 2 s default
    prev = moe.set_wait_limit(12345)
    try:
        assert prev == 2_000_000_000
        assert moe.set_wait_limit(777) == 12345
        assert moe.set_wait_limit(0) == 777
        assert moe.set_wait_limit(-5) == 2_000_000_000
    finally:
        moe.set_wait_limit(prev)
    assert moe.set_wait_limit(0) == 2_000_000_000


def test_error_strings():
    assert moe.error_string(0) == "ok"
    for code in range(1, 7):
        assert moe.error_string(code) not in ("ok", "unknown error")
    assert moe.error_string(99) == "unknown error"


def test_permuted_rows_and_padding_validation():
    p = moe.problem(100, 64, 64, 8, 2)
    assert moe.permuted_rows(p) == 200
    p = moe.problem(100, 64, 64, 8, 2, pad_rows=128)
    assert moe.permuted_rows(p) == 200 + 8 * 127
    lay = moe.workspace_layout(p)
    assert lay["h"] - lay["xp"] >= (200 + 8 * 127) * 64 * 2
    fake = ctypes.c_void_p(1 << 20)
    for bad in (32, 100, 256, -1):
        q = moe.problem(16, 64, 64, 4, 2, pad_rows=bad)
        assert moe.lib.moe_forward(ctypes.byref(q), *([fake] * 11), fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
        assert moe.lib.moe_permuted_rows(ctypes.byref(q)) == 0
    q = moe.problem(16, 64, 64, 4, 2, pad_rows=64)
    assert moe.lib.moe_permute_noalloc(ctypes.byref(q), *([fake] * 7), None) == moe.MOE_ERR_UNSUPPORTED


def test_stats_size_matches_header_layout():
    assert moe.stats_size(8) == 48 + 16 * 8
    assert moe.stats_size(256) == 48 + 16 * 256


def test_workspace_layout_is_aligned_and_ordered():
    for p in (moe.problem(4096, 4096, 14336, 8, 2), moe.problem(8192, 7168, 2048, 256, 8, d_ff_shared=2048),
              moe.problem(1, 128, 256, 8, 2, dtype="f32"), moe.problem(0, 64, 64, 4, 1)):
        lay = moe.workspace_layout(p)
        offs = [lay[n] for n in ("idx", "gate", "pos", "indptr", "row_token", "logits", "xp", "h", "o", "hs", "s")]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs)
        assert lay["total"] == moe.workspace_size(p) >= offs[-1]
    # permuted buffers hold T*k rows
    p = moe.problem(4096, 4096, 14336, 8, 2)
    lay = moe.workspace_layout(p)
    assert lay["h"] - lay["xp"] >= 4096 * 2 * 4096 * 2
    assert lay["o"] - lay["h"] >= 4096 * 2 * 14336 * 2


@pytest.mark.parametrize("kw,code", [
    (dict(T=16, d=64, d_ff=64, E=4, k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(T=16, d=64, d_ff=64, E=4, k=5), moe.MOE_ERR_INVALID_ARG),
    (dict(T=16, d=64, d_ff=64, E=600, k=2), moe.MOE_ERR_INVALID_ARG),
    (dict(T=16, d=64, d_ff=64, E=32, k=17), moe.MOE_ERR_INVALID_ARG),
    (dict(T=-1, d=64, d_ff=64, E=4, k=2), moe.MOE_ERR_INVALID_ARG),
    (dict(T=16, d=96, d_ff=64, E=4, k=2), moe.MOE_ERR_UNSUPPORTED),        # bf16 needs d % 64 == 0
    (dict(T=16, d=64, d_ff=96, E=4, k=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(T=16, d=64, d_ff=64, E=4, k=2, d_ff_shared=32), moe.MOE_ERR_UNSUPPORTED),
    (dict(T=16, d=12, d_ff=64, E=4, k=2, dtype="f32"), moe.MOE_ERR_UNSUPPORTED),  # f32 needs d % 8
])
def test_problem_validation(kw, code):
    p = moe.problem(**kw)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any launch
    rc = moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), fake, 1 << 30, None)
    assert rc == code
    assert moe.lib.moe_workspace_size(ctypes.byref(p)) == 0


def test_bad_bias_mode_and_dtype_rejected():
    p = moe.problem(16, 64, 64, 4, 2)
    p.bias_mode = 7
    fake = ctypes.c_void_p(1 << 20)
    assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    p = moe.problem(16, 64, 64, 4, 2)
    p.dtype = 5
    assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG


def test_bad_gate_and_drop_modes_rejected():
    fake = ctypes.c_void_p(1 << 20)
    for kw, code in ((dict(gate_mode=2), moe.MOE_ERR_INVALID_ARG), (dict(drop_order=5), moe.MOE_ERR_INVALID_ARG),
                     (dict(drop_order=moe.DROP_SLOT), moe.MOE_ERR_UNSUPPORTED)):
        E, k = (512, 16) if kw.get("drop_order") == moe.DROP_SLOT else (4, 2)   # slot order: E*k <= 4096
        p = moe.problem(16, 64, 64, E, k, **kw)
        assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), fake, 1 << 30, None) == code
    p = moe.problem(16, 64, 64, 256, 16, drop_order=moe.DROP_SLOT)   # 4096: allowed
    assert moe.lib.moe_workspace_size(ctypes.byref(p)) > 0


def test_null_and_misaligned_pointers_rejected():
    p = moe.problem(16, 64, 64, 4, 2)
    fake = ctypes.c_void_p(1 << 20)
    args = [fake] * 11
    args[0] = None                                       # x missing
    assert moe.lib.moe_forward(ctypes.byref(p), *args, fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    args = [fake] * 11
    args[3] = ctypes.c_void_p((1 << 20) + 8)             # W1 not 16-byte aligned
    assert moe.lib.moe_forward(ctypes.byref(p), *args, fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # bias required when a bias mode is set
    p = moe.problem(16, 64, 64, 4, 2, bias_mode=moe.BIAS_LOGIT)
    args = [fake] * 11
    args[2] = None
    assert moe.lib.moe_forward(ctypes.byref(p), *args, fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # shared expert weights required when d_ff_shared > 0
    p = moe.problem(16, 64, 64, 4, 2, d_ff_shared=64)
    args = [fake] * 11
    args[7] = None
    assert moe.lib.moe_forward(ctypes.byref(p), *args, fake, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG


def test_small_or_missing_workspace_rejected():
    p = moe.problem(16, 64, 64, 4, 2)
    need = moe.workspace_size(p)
    fake = ctypes.c_void_p(1 << 20)
    assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), fake, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), None, need, None) == moe.MOE_ERR_WORKSPACE
    misaligned = ctypes.c_void_p((1 << 20) + 16)
    assert moe.lib.moe_forward(ctypes.byref(p), *([fake] * 11), misaligned, need, None) == moe.MOE_ERR_WORKSPACE


def test_binding_refuses_cpu_tensors():
    import torch
    p = moe.problem(4, 64, 64, 4, 2)
    t = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.combine(p, t, t, t, t)


def test_gemm_variant_follows_the_shape():
    # host-side selection only (no launch): CTA pairs for prefill-sized
    # experts, GEMVs for GEMM 1/3 of decode batches of at most 8 rows, split-K
    # up to 128 rows, CUDA cores for fp32
    from mixture_experts_layer_62_b200 import inputs

    def variant(name, **kw):
        c = dict(inputs.workload(name), **kw)
        return moe.gemm_variant(moe.problem(c["T"], c["d"], c["d_ff"], c["E"], c["k"], c["cf"], c["dtype"],
                                            c["bias_mode"], c["d_ff_shared"], train=kw.get("train", 0)))
    assert variant("mixtral_prefill") == "pair"
    assert variant("skewed_capacity") == "pair"
    assert variant("decode_t1") == "gemv"
    assert variant("decode_t4") == "gemv"                          # 8 rows
    assert variant("decode_t8") == "split_k"                       # 16 rows
    assert variant("decode_t1", d_ff_shared=1024) == "single"      # a shared expert: ordinary tiles
    assert variant("toy_fp32") == "simt"
    assert variant("mixtral_prefill", T=1000) == "single"          # 250 rows per expert
    assert variant("mixtral_prefill", d_ff=14336, train=1) == "single"
    assert variant("deepseek_v3") == "single"                      # the two-class schedules are opt-in
    with pytest.raises(moe.MoEError):
        moe.gemm_variant(moe.problem(16, 256, 64, 4, 5))            # k > E


def test_router_variant_follows_the_shape():
    # host-side selection only (no launch): the fused router's MMA form for
    # bf16 rows within its shared-memory budget, its FMA form for fp32 and
    # wider rows, tensor cores for wide bf16 routers, the small-batch router
    # in moe_forward for decode-sized batches
    from mixture_experts_layer_62_b200 import inputs

    def variant(name, forward=True, **kw):
        c = dict(inputs.workload(name), **kw)
        return moe.router_variant(moe.problem(c["T"], c["d"], c["d_ff"], c["E"], c["k"], c["cf"], c["dtype"],
                                              c["bias_mode"], c["d_ff_shared"]), forward)
    assert variant("mixtral_prefill") == "fused_mma"
    assert variant("skewed_capacity") == "fused_mma"
    assert variant("decode_t1") == "small"
    assert variant("decode_t1", forward=False) == "fused_mma"      # moe_route has no small-batch path
    assert variant("deepseek_v3") == "tensor"                      # 256 experts
    assert variant("toy_fp32") == "fused_fma"
    assert variant("mixtral_prefill", d=5312) == "fused_mma"       # W_r^T of 8 experts: 84.5 KB
    assert variant("mixtral_prefill", d=5376) == "fused_fma"       # 85.5 KB: past the MMA form's budget
    assert variant("mixtral_prefill", E=72) == "simt"              # wide, but E % 32 != 0
    assert variant("toy_fp32", E=72) == "simt"
    with pytest.raises(moe.MoEError):
        moe.router_variant(moe.problem(16, 256, 64, 4, 5))          # k > E


def test_router_mma_switch_selects_the_fma_form():
    # MOE_ROUTER_MMA=0 is read once per process: checked in a child
    code = ("import mixture_experts_layer_62_b200 as moe; "
            "print(moe.router_variant(moe.problem(4096, 4096, 14336, 8, 2, 0.0, 'bf16'), False))")
    env = dict(os.environ, MOE_ROUTER_MMA="0")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "fused_fma"


def test_debug_library_exports_the_same_entry_points():
    # libmoe_debug.so (device-side bounds checks) is a drop-in for libmoe.so
    from mixture_experts_layer_62_b200 import build as mb
    assert os.path.exists(mb.DEBUG_LIB_PATH), "build() makes the debug library too"
    out = subprocess.run(["nm", "-D", "--defined-only", mb.DEBUG_LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(moe_\w+)", out))
    assert exported == set(declared_functions())
    dbg = ctypes.CDLL(mb.DEBUG_LIB_PATH)
    dbg.moe_error_string.restype = ctypes.c_char_p
    assert dbg.moe_error_string(6).decode() == "device-side bounds check failed (debug build)"
    assert moe.error_string(6) == "device-side bounds check failed (debug build)"
