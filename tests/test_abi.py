"""The C ABI library on the CPU: it builds, loads without a GPU, exports every
function include/pa.h declares, and its host-side checks and helpers behave
as documented.  No kernel is launched here."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

import paged_kv_cache_449_b200 as pa
from paged_kv_cache_449_b200 import build as pabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions(headers=None):
    """Entry points declared in include/*.h (all but the test hooks' pa_test.h
    unless `headers` names the files)."""
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h") and (h in headers if headers else h != "pa_test.h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return set(re.findall(r"\bT\s+(\w+)$", out, flags=re.M))


@pytest.fixture(scope="module")
def lib():
    pabuild.build()
    return pa.load()


def test_header_declares_the_boundary():
    assert declared_functions() == sorted([
        "pa_copy_blocks", "pa_decode", "pa_decode_append", "pa_decode_append_fp8", "pa_decode_fp8", "pa_decode_splitk",
        "pa_decode_splitk_fp8", "pa_decode_splitk_workspace_size", "pa_reshape_and_cache_fp8", "pa_prefill",
        "pa_decode_splitk_static", "pa_get_device_error",
        "pa_reshape_and_cache", "pa_status_string",
        "pa_blocks_init", "pa_blocks_append", "pa_blocks_fork", "pa_blocks_release",
        "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size"])


def declared_signatures():
    """(name, return type, [parameter declarations]) of every entry point in
    include/pa.h, comments stripped."""
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "pa.h")).read(), flags=re.S)
    out = []
    for m in re.finditer(r"^\s*((?:const\s+)?\w+\s*\*?)\s*(pa_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M):
        params = [" ".join(x.split()) for x in m.group(3).split(",") if x.strip() and x.strip() != "void"]
        out.append((m.group(2), " ".join(m.group(1).split()), params))
    return out


def test_binding_argument_types_match_the_header(lib):
    """Every ctypes declaration of the binding has the header's arity, a
    pointer where the header has one and the same scalar type elsewhere, so
    the binding cannot drift from the C ABI."""
    c = ctypes
    scalar = {"int": c.c_int, "int64_t": c.c_int64, "float": c.c_float, "size_t": c.c_size_t,
              "pa_dtype": c.c_int, "pa_status": c.c_int}
    sigs = declared_signatures()
    assert sorted(n for n, _, _ in sigs) == declared_functions()
    for name, ret, params in sigs:
        fn = getattr(lib, name)
        assert fn.argtypes is not None and len(fn.argtypes) == len(params), name
        for decl, ct in zip(params, fn.argtypes):
            if "*" in decl:
                assert ct is c.c_void_p or issubclass(ct, c._Pointer), (name, decl, ct)
            else:
                assert ct is scalar[decl.rsplit(" ", 1)[0].replace("const ", "")], (name, decl, ct)
        assert fn.restype is (c.c_char_p if ret == "const char*" else c.c_int), name


def test_library_exports_every_declared_symbol(lib):
    have = exported(pa.library_path())
    for name in declared_functions():
        assert name in have, name
        assert getattr(lib, name) is not None
    # the test hooks are not in the product library
    hooks = declared_functions(headers=("pa_test.h",))
    assert hooks == ["pa_test_set_hooks", "pa_test_wait_timeout"]
    assert not set(hooks) & have


def test_test_library_exports_the_hooks():
    path = pabuild.build_test()
    have = exported(path)
    for name in declared_functions() + declared_functions(headers=("pa_test.h",)):
        assert name in have, name


def test_library_needs_no_cuda_driver_or_shared_cudart(lib):
    deps = subprocess.run(["ldd", pa.library_path()], capture_output=True, text=True).stdout
    assert "libcuda.so" not in deps and "libcudart.so" not in deps


def test_status_strings(lib):
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(3) == "PA_ERR_WORKSPACE"
    assert pa.pa_status_string(99) == "PA_UNKNOWN_STATUS"


def test_workspace_size(lib):
    # S * Hq * ceil(max_len / part) * (D + 2) * 4 bytes
    assert pa.pa_decode_splitk_workspace_size(32, 64, 128, 32768, 512) == 32 * 64 * 64 * 130 * 4
    assert pa.pa_decode_splitk_workspace_size(4, 4, 64, 100, 512) == 4 * 4 * 1 * 66 * 4
    assert pa.pa_decode_splitk_workspace_size(4, 4, 64, 0, 512) == 0
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_decode_splitk_workspace_size(4, 4, 64, 100, 0)


P = ctypes.c_void_p


def _decode(lib, **kw):
    a = dict(out=16, q=16, k=16, v=16, bt=16, cl=16, scale=0.125, B=16, S=4, Hq=4, Hkv=4, D=64, mb=7, mcl=100,
             N=64, dt=0, order=None)
    a.update(kw)
    return lib.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["scale"], a["B"], a["S"], a["Hq"],
                         a["Hkv"], a["D"], a["mb"], a["mcl"], a["N"], a["dt"], a["order"], None)


def test_host_validation_rejects_before_launch(lib):
    # Every case here fails validation, so nothing reaches the (absent) GPU.
    assert _decode(lib, D=96) == 2                 # unsupported head_dim
    assert _decode(lib, B=12) == 2                 # unsupported block_size
    assert _decode(lib, Hq=12, Hkv=4) == 2         # group 3
    assert _decode(lib, Hq=6, Hkv=4) == 1          # not a multiple
    assert _decode(lib, dt=7) == 2                 # unknown dtype
    assert _decode(lib, q=0) == 1                  # null pointer
    assert _decode(lib, k=24) == 1                 # misaligned pool
    assert _decode(lib, N=0) == 1                  # empty pool
    assert _decode(lib, scale=float("nan")) == 1
    assert _decode(lib, S=0) == 0                  # empty batch: a no-op
    assert _decode(lib, order=18) == 1             # misaligned seq_order
    assert lib.pa_reshape_and_cache(16, 16, 16, 16, 16, 4, 8, 100, 16, 10, 2, None) == 2   # 200 B rows
    assert lib.pa_reshape_and_cache(16, 16, 16, 16, 12, 4, 8, 128, 16, 10, 2, None) == 1   # slots misaligned
    assert lib.pa_reshape_and_cache(0, 0, 0, 0, 0, 0, 8, 128, 16, 10, 2, None) == 0        # no tokens
    args = [16, 16, 16, 16, 16, 16, 0.125, 16, 4, 4, 4, 64, 7, 100, 64, 0]
    assert lib.pa_decode_splitk(*args, 500, 16, 1 << 20, None, 0, None, None) == 1   # partition not a multiple of 16
    assert lib.pa_decode_splitk(*args, 512, 16, 100, None, 0, None, None) == 3       # workspace too small
    assert lib.pa_decode_splitk(*args, 512, 0, 1 << 20, None, 0, None, None) == 3    # no workspace
    assert lib.pa_decode_splitk(*args, 512, 16, 1 << 20, 16, 3, None, None) == 3     # too few counters
    assert lib.pa_decode_splitk(*args, 512, 16, 1 << 20, None, 0, 6, None) == 1      # misaligned seq_order
    assert lib.pa_decode_append(16, 16, 16, 16, *args[2:], None, 2, None) == 1      # misaligned seq_order
    assert lib.pa_decode_append(16, 16, 16, 16, *args[2:], 6, None, None) == 1      # misaligned ref_counts
    # shared prefix: S 4, Hq 4, D 64, prefix 3 blocks of 16 (one 64-key tile + the own-block partial):
    # 4*4*2*66*4 bytes of workspace; counters for S * Hkv = 16 (sequence, kv head) pairs
    sp = [16, 16, 16, 16, 16, 16, 16, 16, 0.125, 16, 4, 4, 4, 64, 7, 100, 64, 1]
    ws = 4 * 4 * 2 * 66 * 4
    size = ctypes.c_size_t(0)
    assert lib.pa_decode_shared_prefix_workspace_size(4, 4, 64, 3, 16, ctypes.byref(size)) == 0 and size.value == ws
    cn = [16, 16]
    assert lib.pa_decode_shared_prefix(*sp[:17], 0, 3, 16, ws, *cn, None, None) == 2          # fp32
    assert lib.pa_decode_shared_prefix(*sp, 0, 16, ws, *cn, None, None) == 1                  # no prefix
    assert lib.pa_decode_shared_prefix(*sp, 8, 16, ws, *cn, None, None) == 1                  # more than a row holds
    assert lib.pa_decode_shared_prefix(*sp[:3], None, *sp[4:], 3, 16, ws, *cn, None, None) == 1   # key, no value
    assert lib.pa_decode_shared_prefix(*sp, 3, 16, ws - 1, *cn, None, None) == 3              # workspace too small
    assert lib.pa_decode_shared_prefix(*sp, 3, 24, ws, *cn, None, None) == 3                  # misaligned workspace
    assert lib.pa_decode_shared_prefix(*sp, 3, 16, ws, None, 16, None, None) == 3             # no counters
    assert lib.pa_decode_shared_prefix(*sp, 3, 16, ws, 16, 15, None, None) == 3               # too few counters
    assert lib.pa_decode_shared_prefix(*sp, 3, 16, ws, 18, 16, None, None) == 3               # misaligned counters
    assert lib.pa_decode_shared_prefix(*sp, 3, 16, ws, *cn, 6, None) == 1                     # misaligned ref_counts
    cp = [16, 16, 16, 16, 16, 4, 8, 128, 16, 10, 10, 2, None]
    assert lib.pa_copy_blocks(*cp[:5], 0, *cp[6:]) == 0                             # no pairs: a no-op
    assert lib.pa_copy_blocks(*cp[:5], -1, *cp[6:]) == 1                            # negative count
    assert lib.pa_copy_blocks(0, *cp[1:]) == 1                                      # null pool
    assert lib.pa_copy_blocks(*cp[:4], 12, *cp[5:]) == 1                            # mapping not 8-byte aligned
    assert lib.pa_copy_blocks(*cp[:2], 24, *cp[3:]) == 1                            # pool not 16-byte aligned
    assert lib.pa_copy_blocks(*cp[:7], 100, *cp[8:]) == 2                           # 200-byte rows
    assert lib.pa_copy_blocks(*cp[:9], 0, *cp[10:]) == 1                            # empty source pool
    f8 = [16, 16, 16, 16, 16, 16, 16, 16, 0.125, 16, 4, 4, 4, 64, 7, 100, 64]
    assert lib.pa_decode_fp8(*f8, 0, None, None) == 2                                # fp32 queries
    assert lib.pa_decode_append_fp8(16, 16, 0, 16, *f8[2:], 2, None, None, None) == 1      # no new key
    assert lib.pa_decode_append_fp8(16, 16, 16, 16, *f8[2:], 0, None, None, None) == 2     # fp32 queries
    assert lib.pa_decode_append_fp8(16, 16, 16, 16, *f8[2:], 2, 6, None, None) == 1       # misaligned ref_counts
    assert lib.pa_decode_fp8(*f8[:4], 0, *f8[5:], 2, None, None) == 1                # no K scale
    assert lib.pa_decode_fp8(*f8[:5], 18, *f8[6:], 2, None, None) == 1               # V scale misaligned
    assert lib.pa_decode_splitk_fp8(*f8, 1, 500, 16, 1 << 20, None, 0, None, None) == 1  # partition not x16
    assert lib.pa_decode_splitk_fp8(*f8, 1, 512, 16, 100, None, 0, None, None) == 3       # workspace too small
    assert lib.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 16, 16, 4, 8, 40, 16, 10, 2, None) == 2  # D % 16
    assert lib.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 0, 16, 4, 8, 64, 16, 10, 2, None) == 1   # no scale
    # block management: refused before any launch
    assert lib.pa_blocks_init(16, 16, 16, 0, None) == 1                                 # no blocks
    assert lib.pa_blocks_init(16, 16, 12, 8, None) == 1                                 # state not 8-byte aligned
    assert lib.pa_blocks_init(16, 0, 16, 8, None) == 1                                  # no ring
    ap = [16, 16, 16, 16, 16, 16, 16, 4, 16, 4, 8, 16, 64, None]
    assert lib.pa_blocks_append(*ap[:9], 0, *ap[10:]) == 0                              # no sequences: no-op
    assert lib.pa_blocks_append(*ap[:8], 12, *ap[9:]) == 1                              # pairs not 8-byte aligned
    assert lib.pa_blocks_append(*ap[:7], -1, *ap[8:]) == 1                              # negative slot capacity
    assert lib.pa_blocks_append(*ap[:11], 0, *ap[12:]) == 1                             # block size 0
    assert lib.pa_blocks_append(*ap[:12], 1 << 40, None) == 1                           # more blocks than int32 ids
    assert lib.pa_blocks_fork(16, 16, 16, 16, 0, 4, 8, 16, 64, None) == 0               # no forks: no-op
    assert lib.pa_blocks_fork(16, 16, 16, 18, 2, 4, 8, 16, 64, None) == 1               # forks misaligned
    assert lib.pa_blocks_release(16, 16, 16, 16, 16, 16, -1, 4, 8, 16, 64, None) == 1   # negative count
    assert lib.pa_blocks_release(16, 16, 16, 16, 16, 0, 2, 4, 8, 16, 64, None) == 1     # no list
    pf = [16, 16, 16, 16, 16, 16, 16, 0.125, 16, 4, 4, 4, 64, 7, 100, 100, 64]
    assert lib.pa_prefill(*pf, 0, None) == 2                                             # fp32 queries
    assert lib.pa_prefill(*pf[:6], 0, *pf[7:], 2, None) == 1                             # no query_start
    assert lib.pa_prefill(*pf[:15], -1, 64, 2, None) == 1                                # negative max query
    assert lib.pa_prefill(*pf[:15], 0, 64, 2, None) == 0                                 # no queries: no-op


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(pa, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(pa, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        pa.load()


def test_longest_first_is_a_stable_descending_permutation():
    import torch
    lens = torch.tensor([5, 300, 17, 300, 0, 64], dtype=torch.int32)
    order = pa.longest_first(lens)
    assert order.dtype == torch.int32
    assert order.tolist() == [1, 3, 5, 2, 0, 4]
    assert pa.longest_first([]).numel() == 0


class _FakeCudaTensor(torch.Tensor):
    """A CPU tensor that reports a CUDA device: enough for the binding's
    device check, which runs before anything reaches the library."""

    @staticmethod
    def make(index):
        t = torch.Tensor._make_subclass(_FakeCudaTensor, torch.zeros(4))
        t.fake_device = torch.device("cuda", index)
        return t

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return self.fake_device


def test_binding_refuses_tensors_on_two_devices():
    a, b = _FakeCudaTensor.make(0), _FakeCudaTensor.make(1)
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_decode(a, b, a, a, a, a, 0.125)
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_reshape_and_cache(a, a, a, a, slot_mapping=b)
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.pa_decode_splitk_static(a, a, a, a, a, b, 0.125, 64)
    assert pa._tensor_device((a, 3, None), {"x": a}) == torch.device("cuda", 0)
    assert pa._tensor_device((torch.zeros(2),), {}) is None


# every entry point that takes tensors, with its number of leading tensor arguments
TENSOR_ENTRIES = {
    "pa_reshape_and_cache": 5, "pa_decode": 6, "pa_decode_append": 8, "pa_decode_splitk": 6,
    "pa_decode_splitk_static": 6, "pa_copy_blocks": 5, "pa_reshape_and_cache_fp8": 7, "pa_decode_fp8": 8,
    "pa_decode_append_fp8": 10, "pa_decode_splitk_fp8": 8, "pa_prefill": 7, "pa_blocks_init": 3,
    "pa_blocks_append": 7, "pa_blocks_fork": 4, "pa_blocks_release": 6, "pa_decode_shared_prefix": 8,
}


def test_every_tensor_entry_checks_the_device():
    """Each tensor entry point runs under the device guard (a helper may not
    take its place) and refuses tensors on two devices before any marshalling."""
    public = {n for n in dir(pa) if n.startswith("pa_") and callable(getattr(pa, n))}
    takes_tensors = public - {"pa_status_string", "pa_get_device_error", "pa_decode_splitk_workspace_size",
                              "pa_decode_shared_prefix_workspace_size"}
    assert takes_tensors == set(TENSOR_ENTRIES)
    a, b = _FakeCudaTensor.make(0), _FakeCudaTensor.make(1)
    for name, n in TENSOR_ENTRIES.items():
        fn = getattr(pa, name)
        assert getattr(fn, "__wrapped__", None) is not None, name
        args = [a] * (n - 1) + [b]
        with pytest.raises(ValueError, match="one CUDA device"):
            fn(*args, *([0] * 8))
    for fn, n in ((pa.prepare_decode_append, 8), (pa.prepare_decode_append_fp8, 10)):
        with pytest.raises(ValueError, match="one CUDA device"):
            fn(*([a] * (n - 1) + [b]), 0.125)
    with pytest.raises(ValueError, match="one CUDA device"):
        pa.prepare_decode_shared_prefix(*([a] * 7 + [b]), 0.125, 4)
    with pytest.raises(ValueError, match="CUDA tensors"):
        pa.prepare_decode_append(*([torch.zeros(2)] * 8), 0.125)
    with pytest.raises(ValueError, match="CUDA tensors"):
        pa.prepare_decode_shared_prefix(*([torch.zeros(2)] * 8), 0.125, 4)
