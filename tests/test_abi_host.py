"""C ABI: symbols and host-side argument checks (CPU only).

Every mla_decode call here is invalid in a way the library detects before it
touches the device, so the fake pointers are never dereferenced (this file is
also safe to run on a GPU machine).
"""
import ctypes
import os
import re

import pytest

import mla_paged_decode_04_b200 as mla
from mla_paged_decode_04_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(mla_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert "mla_decode" in names and "mla_decode_plan" in names
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(_lib.EXPORTED)


def test_bounds_checking_build_exports_the_same_symbols():
    """libmla_decode_check.so (MLA_BOUNDS_CHECK=1) declares nothing else and says which it is."""
    names = _declared_functions()
    check = _lib.load_library(_lib.CHECK_LIB_PATH)
    for n in names:
        assert hasattr(check, n), n
    assert check.mla_bounds_checked() == 1
    assert _lib.load_library(_lib.NORMAL_LIB_PATH).mla_bounds_checked() == 0
    assert "mla_bounds_checked" in names


def test_store_fault_mode_exists_in_the_checking_build_only():
    """fault_test = 2 (stores past the buffers) is refused before any launch by the normal build;
    the checking build accepts it on the FP8 CTA-pair kernel's balanced plans only."""
    fp8 = mla.mla_decode_plan(2, 4, 32, 256, "fp8")
    bf16 = mla.mla_decode_plan(2, 4, 32, 256, "bf16")
    bad = _lib.MlaPlan.from_buffer_copy(fp8)
    bad.fault_test = 2
    assert _call(bad, lib=_lib.load_library(_lib.NORMAL_LIB_PATH)) == -6
    check = _lib.load_library(_lib.CHECK_LIB_PATH)
    bad16 = _lib.MlaPlan.from_buffer_copy(bf16)
    bad16.fault_test = 2
    assert _call(bad16, lib=check) == -6
    # accepted: the call then fails only on the fake (host-side refused) workspace size
    assert _call(bad, lib=check, ws_bytes=0) == -3


def test_library_is_built_for_sm100a():
    # the build records ptxas reports per translation unit
    build = os.path.join(ROOT, "_build")
    logs = [f for f in os.listdir(build) if f.endswith(".ptxas.txt")]
    assert logs
    text = "".join(open(os.path.join(build, f)).read() for f in logs)
    assert "for 'sm_100a'" in text and "spill stores" in text


def test_status_strings_and_version():
    assert mla.status_string(0) == "MLA_OK"
    assert mla.status_string(-3) == "MLA_ERR_WORKSPACE_TOO_SMALL"
    assert mla.status_string(-99) == "MLA_ERR_UNKNOWN"
    assert mla.mla_version().count(".") == 2


FAKE = 1 << 20  # 256-byte aligned, never dereferenced


def _call(plan, **kw):
    args = dict(q=FAKE, kv=FAKE, num_pages=8, page_size=64, bt=FAKE, maxp=4, sl=FAKE,
                scale=0.04, qs=1.0, ks=1.0, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30)
    L = kw.pop("lib", None) or _lib.lib()
    args.update(kw)
    vp = ctypes.c_void_p
    return L.mla_decode(ctypes.byref(plan) if plan is not None else None, vp(args["q"]),
                        vp(args["kv"]), args["num_pages"], args["page_size"], vp(args["bt"]),
                        args["maxp"], vp(args["sl"]), args["scale"], args["qs"], args["ks"],
                        vp(args["out"]), vp(args["lse"]), vp(args["ws"]), args["ws_bytes"], None)


def test_decode_rejects_bad_arguments_before_any_launch():
    p = mla.mla_decode_plan(2, 4, 32, 256, "fp8")
    assert _call(None) == -6
    bad = _lib.MlaPlan.from_buffer_copy(p)
    bad.magic = 0
    assert _call(bad) == -6
    bad = _lib.MlaPlan.from_buffer_copy(p)
    bad.fold = 3
    assert _call(bad) == -6
    bad = _lib.MlaPlan.from_buffer_copy(p)
    bad.keys_per_split = 64
    bad.split_kv = 1  # no longer covers max_seq_len
    assert _call(bad) == -6
    assert _call(p, page_size=32) == -2
    assert _call(p, ws=0) == -1
    assert _call(p, ws=FAKE + 16) == -1           # workspace not 256-aligned
    assert _call(p, ws_bytes=p.workspace_bytes - 1) == -3
    assert _call(p, q=0) == -1
    assert _call(p, kv=0) == -1
    assert _call(p, bt=0) == -1
    assert _call(p, sl=0) == -1
    assert _call(p, out=0) == -1
    assert _call(p, q=FAKE + 8) == -1             # q not 16-byte aligned
    assert _call(p, num_pages=0) == -1
    assert _call(p, maxp=0) == -1
    assert _call(p, qs=0.0) == -1                 # FP8 scales must be positive
    assert _call(p, ks=float("nan")) == -1
    assert _call(p, scale=float("inf")) == -1


def test_fault_test_mode_is_off_in_plans_and_refused_where_it_does_not_exist():
    """The failure-detection test field is 0 in every plan the planner writes; 1 is accepted only on
    the FP8 CTA-pair kernel's balanced plans, anything else is refused before any launch."""
    fp8 = mla.mla_decode_plan(2, 4, 32, 256, "fp8")
    bf16 = mla.mla_decode_plan(2, 4, 32, 256, "bf16")
    simt = mla.mla_decode_plan_custom(2, 4, 32, 256, "fp8", kernel="simt")
    assert fp8.fault_test == 0 and bf16.fault_test == 0 and simt.fault_test == 0
    for plan, value in ((bf16, 1), (simt, 1), (fp8, 2), (fp8, -1)):
        bad = _lib.MlaPlan.from_buffer_copy(plan)
        bad.fault_test = value
        assert _call(bad) == -6


def test_python_wrapper_refuses_host_tensors():
    """The binding names the first argument that is not a CUDA tensor before calling the library."""
    torch = pytest.importorskip("torch")
    p = mla.mla_decode_plan(1, 1, 16, 256, "bf16")
    t = torch.empty(0)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        mla.mla_decode(p, t, torch.empty(1, 32, 576), torch.empty(1, 4, dtype=torch.int32), t,
                       0.04, t, None, torch.empty(0, dtype=torch.uint8))


def test_prefill_wrapper_refuses_host_tensors():
    torch = pytest.importorskip("torch")
    p = mla.mla_prefill_plan(1, 4, 16, 256, "bf16")
    t = torch.empty(0)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        mla.mla_prefill(p, t, torch.zeros(2, dtype=torch.int32), torch.empty(1, 64, 576),
                        torch.empty(1, 4, dtype=torch.int32), t, 0.04, t, None, torch.empty(0, dtype=torch.uint8))


def test_last_cuda_error_starts_clean():
    """No CUDA failure has been recorded on a fresh thread: code 0, name cudaSuccess."""
    import threading
    res = {}
    t = threading.Thread(target=lambda: res.setdefault("v", mla.last_cuda_error()))
    t.start()
    t.join()
    assert res["v"] == (0, "cudaSuccess")


def test_decode_rejects_a_window_the_plan_cannot_run():
    """A window written into a plan by hand is checked like every other plan field."""
    p = mla.mla_decode_plan(2, 4, 32, 256, "fp8")
    bad = _lib.MlaPlan.from_buffer_copy(p)
    bad.window = -4
    assert _call(bad) == -6
    solo = mla.mla_decode_plan_custom(2, 4, 32, 256, "fp8", kernel="tcgen05_solo")
    bad = _lib.MlaPlan.from_buffer_copy(solo)
    bad.window = 64
    assert _call(bad) == -6


def _prefill_call(plan, cu=FAKE, total_q=8, **kw):
    args = dict(q=FAKE, kv=FAKE, num_pages=8, page_size=64, bt=FAKE, maxp=4, sl=FAKE,
                scale=0.04, qs=1.0, ks=1.0, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30)
    args.update(kw)
    vp = ctypes.c_void_p
    return _lib.lib().mla_prefill(ctypes.byref(plan), vp(args["q"]), total_q, vp(cu), vp(args["kv"]),
                                  args["num_pages"], args["page_size"], vp(args["bt"]), args["maxp"],
                                  vp(args["sl"]), args["scale"], args["qs"], args["ks"], vp(args["out"]),
                                  vp(args["lse"]), vp(args["ws"]), args["ws_bytes"], None)


def test_prefill_and_decode_refuse_each_others_plans():
    pre = mla.mla_prefill_plan(2, 4, 32, 256, "fp8")
    dec = mla.mla_decode_plan(2, 4, 32, 256, "fp8")
    assert _call(pre) == -6                  # a ragged plan needs cu_seqlens_q
    assert _prefill_call(dec) == -6          # a decode plan has no ragged queries
    assert _prefill_call(pre, cu=0) == -1    # null cu_seqlens_q
    assert _prefill_call(pre, total_q=9) == -1   # more tokens than batch x max_q_len
    assert _prefill_call(pre, total_q=-1) == -1
    assert _prefill_call(pre, cu=FAKE + 2) == -1  # cu_seqlens_q not 4-byte aligned
    bad = _lib.MlaPlan.from_buffer_copy(pre)
    bad.varlen = 2
    assert _prefill_call(bad) == -6
    bad = _lib.MlaPlan.from_buffer_copy(pre)
    bad.kernel = 3  # the solo kernel has no ragged form
    assert _prefill_call(bad) == -6
