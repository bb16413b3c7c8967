"""Host-side checks of the C ABI: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from lsh_attention_02_b200 import build as lib_build
import lsh_attention_02_b200 as lsh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsh_attn.h")


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return lsh.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LSH_API\s+[\w\s\*]+?\b(lsh_attn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ["lsh_attn_fwd", "lsh_attn_bwd", "lsh_attn_workspace_size", "lsh_attn_hash", "lsh_attn_sort",
              "lsh_attn_fwd_sorted", "lsh_attn_status_str"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(lsh.EXPORTED)


def test_abi_version(lib):
    text = open(HEADER).read()
    v = int(re.search(r"#define LSH_ATTN_ABI_VERSION (\d+)", text).group(1))
    assert lib.lsh_attn_abi_version() == v


def test_status_strings(lib):
    for code in lsh.STATUS:
        s = lib.lsh_attn_status_str(code)
        assert s and isinstance(s, bytes)
    assert lib.lsh_attn_status_str(42) == b"unknown status"


def _desc(**kw):
    base = dict(B=1, H=2, L=1024, d=64, n_buckets=16, n_hashes=2, chunk=64, causal=0, dtype=lsh.LSH_BF16,
                flags=0)
    base.update(kw)
    return lsh.Desc(*[base[k] for k in ("B", "H", "L", "d", "n_buckets", "n_hashes", "chunk", "causal", "dtype",
                                        "flags")])


@pytest.mark.parametrize("kw,want", [
    (dict(d=32), -4), (dict(L=1000), -2), (dict(n_buckets=15), -2), (dict(n_buckets=0), -2),
    (dict(n_hashes=0), -2), (dict(chunk=0), -2), (dict(dtype=7), -1), (dict(flags=4), -1), (dict(causal=2), -1),
    (dict(B=0), -2), (dict(n_buckets=131072), -2),
])
def test_invalid_descriptors_rejected(lib, kw, want):
    d = _desc(**kw)
    assert lib.lsh_attn_workspace_size(ctypes.byref(d), 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.lsh_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake, 1 << 40, None)
    assert rc == want


def test_null_and_misaligned_pointers(lib):
    d = _desc()
    ws_n = lib.lsh_attn_workspace_size(ctypes.byref(d), 0)
    assert ws_n > 0
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.lsh_attn_fwd(ctypes.byref(d), None, ok, ok, ok, ok, None, ok, ws_n, None) == -1
    assert lib.lsh_attn_fwd(ctypes.byref(d), bad, ok, ok, ok, ok, None, ok, ws_n, None) == -3
    # workspace: null, misaligned (needs 256 B) and too small
    assert lib.lsh_attn_fwd(ctypes.byref(d), ok, ok, ok, ok, ok, None, None, ws_n, None) == -1
    assert lib.lsh_attn_fwd(ctypes.byref(d), ok, ok, ok, ok, ok, None, ctypes.c_void_p((1 << 20) + 16), ws_n,
                            None) == -3
    assert lib.lsh_attn_fwd(ctypes.byref(d), ok, ok, ok, ok, ok, None, ok, ws_n - 1, None) == -7
    # backward needs either perm or rotations
    wb = lib.lsh_attn_workspace_size(ctypes.byref(d), 1)
    assert lib.lsh_attn_bwd(ctypes.byref(d), ok, ok, None, ok, ok, None, ok, ok, ok, ok, wb, None) == -1
    assert lib.lsh_attn_bwd(ctypes.byref(d), ok, ok, ok, ok, ok, None, ok, ok, ok, ok, wb - 1, None) == -7


def test_workspace_grows_with_problem(lib):
    small = lib.lsh_attn_workspace_size(ctypes.byref(_desc()), 1)
    big = lib.lsh_attn_workspace_size(ctypes.byref(_desc(L=4096)), 1)
    assert 0 < small < big
    # fwd and bwd sizes are positive for both element types
    for dtype in (lsh.LSH_F32, lsh.LSH_BF16):
        for bwd in (0, 1):
            assert lib.lsh_attn_workspace_size(ctypes.byref(_desc(dtype=dtype)), bwd) > 0


@pytest.mark.parametrize("kw", [dict(chunk=32), dict(chunk=128), dict(chunk=1, L=96), dict(B=1, H=1, L=64)])
def test_bf16_outside_tensor_core_envelope_refused(lib, kw):
    """bf16 runs on the tensor-core kernels only (chunk 64, L % 64 == 0, at least
    128 rows): any other bf16 request is refused with LSH_ERR_UNSUPPORTED by every
    computing entry point before anything is launched (the fake pointers are never
    dereferenced), while the same shape in fp32 is accepted by the checks."""
    d = _desc(**kw)
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    assert lib.lsh_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake, big, None) == -4
    assert lib.lsh_attn_fwd_sorted(ctypes.byref(d), fake, fake, fake, fake, fake, fake, big, None) == -4
    assert lib.lsh_attn_hash(ctypes.byref(d), fake, fake, fake, fake, big, None) == -4
    assert lib.lsh_attn_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, big,
                            None) == -4
    assert lib.lsh_attn_workspace_size(ctypes.byref(_desc(**kw, **{"dtype": lsh.LSH_F32})), 0) > 0


def test_trace_end_without_begin_is_an_error(lib):
    n = len(lsh.STAGES)
    ms = (ctypes.c_float * n)(); c = (ctypes.c_int32 * n)(); k = (ctypes.c_int32 * n)()
    assert lib.lsh_attn_trace_end(ms, c, k, n) == -1
    assert lib.lsh_attn_trace_begin(0) == -1


def test_near_tie_count_not_compiled_in_regular_build(lib):
    lib.lsh_attn_last_near_ties.restype = ctypes.c_int
    assert lib.lsh_attn_last_near_ties() == -1


def test_static_sort_rejects_oversize_before_any_device_call(lib):
    """Two-pass sort (65536 buckets) of 32 segments x 131072 positions needs
    24 MiB of scratch, over the 16 MiB limit: refused on the host, with the
    sizes in the error text; the (never dereferenced) pointers are fakes."""
    import lsh_attention_02_b200 as lsh
    desc = lsh.make_desc(1, 32, 131072, 64, 65536, 1, 64, False, lsh.LSH_BF16)
    fake = ctypes.c_void_p(0x1000)
    lib.lsh_attn_sort_static.argtypes = [ctypes.POINTER(lsh.Desc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert lib.lsh_attn_sort_static(ctypes.byref(desc), fake, fake, None) == -7
    lib.lsh_attn_last_error.restype = ctypes.c_char_p
    msg = lib.lsh_attn_last_error().decode()
    assert "lsh_attn_sort_static" in msg and str(16 << 20) in msg


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_flags_accepted_and_their_argument_rules(lib, flags):
    """The optional readings are accepted by the checks; the bucket mask needs
    bucket ids, so lsh_attn_fwd_sorted refuses it and lsh_attn_bwd needs R to
    recompute them (fake pointers, never dereferenced)."""
    d = _desc(flags=flags)
    assert lib.lsh_attn_workspace_size(ctypes.byref(d), 1) > 0
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    if flags & 1:
        assert lib.lsh_attn_fwd_sorted(ctypes.byref(d), fake, fake, fake, fake, fake, fake, big, None) == -1
        assert lib.lsh_attn_bwd(ctypes.byref(d), fake, fake, None, fake, fake, fake, fake, fake, fake, fake, big,
                                None) == -1


def test_local_attention_argument_rules(lib):
    """Local attention: one set of outputs (n_hashes 1), no bucket mask, one or
    no following chunk; n_buckets is not used (fake pointers, never read)."""
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    ok = _desc(n_hashes=1, n_buckets=0)
    assert lib.lsh_attn_local_workspace_size(ctypes.byref(ok), 1, 0) > 0
    assert lib.lsh_attn_local_workspace_size(ctypes.byref(ok), 1, 1) > 0
    assert lib.lsh_attn_local_fwd(ctypes.byref(_desc(n_hashes=2)), 1, fake, fake, fake, fake, fake, big, None) == -2
    assert lib.lsh_attn_local_fwd(ctypes.byref(_desc(n_hashes=1, flags=1)), 1, fake, fake, fake, fake, fake, big,
                                  None) == -1
    assert lib.lsh_attn_local_fwd(ctypes.byref(ok), 2, fake, fake, fake, fake, fake, big, None) == -4
    assert lib.lsh_attn_local_bwd(ctypes.byref(ok), 1, fake, fake, None, fake, fake, fake, fake, fake, big,
                                  None) == -1


def test_fused_forward_applies_to_short_bf16_segments_only(lib):
    """The single-kernel forward is chosen on the host from the descriptor alone.
    Setting 2: wherever it fits (bf16, chunk 64, L a multiple of 64 up to 4096,
    n_buckets <= 128, n_hashes <= 8, B*H*L >= 128).  Setting 1 (the default):
    also only where the B*H*n_hashes segments make one well-filled wave (from
    three quarters of the SM count up to it; without a device the B200's 148).
    Setting 0: never."""
    fits = lambda **kw: lib.lsh_attn_fused_forward_fits(ctypes.byref(_desc(**kw)))
    assert lib.lsh_attn_fused_forward(3) == -1     # LSH_ERR_ARG
    try:
        assert lib.lsh_attn_fused_forward(2) == 0
        assert fits(L=4096, n_buckets=64, n_hashes=2, B=8, H=8, causal=1) == 1
        assert fits(L=64) == 1 and fits(L=960, n_buckets=2) == 1 and fits(n_buckets=128, n_hashes=8) == 1
        assert fits(L=4160) == 0                       # longer than a segment held on chip
        assert fits(n_buckets=130) == 0                # more rotation columns than the kernel holds
        assert fits(n_hashes=9) == 0                   # more rounds than a portable cluster has CTAs
        assert fits(dtype=lsh.LSH_F32) == 0            # fp32 runs on the CUDA-core kernels
        assert fits(chunk=32) == 0 and fits(B=1, H=1, L=64) == 0
        assert lib.lsh_attn_fused_forward(1) == 0
        sms = 148 if not torch_cuda_available() else None
        if sms is not None:
            assert fits(L=4096, n_buckets=64, n_hashes=2, B=8, H=8) == 1    # 128 segments, one wave
            assert fits(L=4096, n_buckets=64, n_hashes=2, B=1, H=2) == 0    # 4 segments: staged
            assert fits(L=1024, n_buckets=64, n_hashes=2, B=8, H=9) == 1    # 144 segments, one wave
            assert fits(L=1024, n_buckets=64, n_hashes=2, B=8, H=10) == 0   # 160 segments: a second wave
            assert fits(L=1024, n_buckets=64, n_hashes=2, B=8, H=16) == 0   # 256 segments: staged
        assert lib.lsh_attn_fused_forward(0) == 0
        assert fits(L=4096, n_buckets=64, B=8, H=8) == 0
    finally:
        assert lib.lsh_attn_fused_forward(1) == 0


def torch_cuda_available():
    import torch
    return torch.cuda.is_available()


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without the CUDA library every entry point raises: there is no other
    implementation to fall back on."""
    absent = str(tmp_path / "liblsh_attn.so")
    monkeypatch.setattr(lsh, "_lib", None)
    monkeypatch.setattr(lsh.load_library, "__defaults__", (absent,))
    with pytest.raises(ImportError, match="missing"):
        lsh.load_library()
    desc = lsh.make_desc(1, 1, 256, 64, 16, 1, 64, True, lsh.LSH_BF16)
    with pytest.raises(ImportError, match="missing"):
        lsh.workspace_size(desc, False)
