"""The C-ABI library loads, exports every symbol include/sage.h declares, and
rejects bad arguments on the host before touching a device (no GPU needed)."""
import ctypes

import pytest

from video_dit_quantized_b200 import sage

EXPECTED = {
    "sage_workspace_bytes", "sage_prepass_scratch_bytes", "sage_quantize_qk", "sage_attn_quantized",
    "sage_attn_fwd", "attn_layer_schedule", "sage_status", "sage_strerror", "sage_device_check",
    "sage_dbg_qk_tiles", "sage_dbg_pv_tile", "sage_dbg_qk_bf16_tile", "sage_dbg_attn_forced_timeout",
    "sage_quantize_qk_noalloc", "sage_attn_fwd_host", "sage_error_scratch_bytes", "sage_attn_error_stats",
    "sage_select_full_precision_layers", "sage_quantize_qk_ex", "sage_attn_quantized_ex",
    "sage_quantize_blocks_2d", "sage_linear_w8a8", "sage_dbg_linear_forced_timeout",
    "sage_dequant_blocks_2d", "sage_linear_bf16", "sage_linear_w8a16_workspace_bytes", "sage_linear_w8a16",
    "sage_ulysses_permute", "sage_host_chunk_heads", "sage_host_workspace_bytes", "sage_dbg_mma_peak", "sage_dbg_linear_bf16_forced_timeout",
    "sage_attn_rel_l2", "sage_seqpar_workspace_bytes", "sage_attn_fwd_seqpar",
    "sage_debug_build", "sage_debug_last_failure", "sage_dbg_bounds_selftest",
}


def test_header_declares_the_expected_entry_points():
    assert set(sage.header_functions()) == EXPECTED


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sage._build.LIB_PATH)
    for name in sage.header_functions():
        assert hasattr(lib, name), name


def test_debug_build_exports_the_same_symbols_and_says_it_is_one():
    dbg = sage.debug_library()
    for name in sage.header_functions():
        assert hasattr(dbg, name), name
    assert sage.LIB.sage_debug_build() == 0 and dbg.sage_debug_build() == 1
    site, index = ctypes.c_int(-1), ctypes.c_longlong(-1)
    # a release build keeps no failure record; a debug build has none yet
    assert sage.LIB.sage_debug_last_failure(ctypes.byref(site), ctypes.byref(index)) == sage.EUNSUPPORTED
    assert dbg.sage_debug_last_failure(ctypes.byref(site), ctypes.byref(index)) == sage.OK
    assert (site.value, index.value) == (0, 0)
    assert dbg.sage_debug_last_failure(None, None) == sage.EINVAL
    # the release self-test has no check to fail; neither touches a device before that answer
    assert sage.LIB.sage_dbg_bounds_selftest(None) == sage.EUNSUPPORTED
    assert sage.strerror(sage.EBOUNDS) == "a device-side bounds check failed (debug build)"


def test_workspace_sizes():
    # BF16 mode needs only the status word
    assert sage.workspace_bytes(1, 2, 1024, 128, sage.MODE_BF16) == 256
    # INT8/FP8: Q_i8 + K_i8 + V_f8t dominate (3 bytes per element of the padded tensor)
    B, H, N, d = 1, 40, 75600, 128
    npad = (N + 127) // 128 * 128
    ws = sage.workspace_bytes(B, H, N, d, sage.MODE_INT8_FP8)
    assert 3 * B * H * npad * d < ws < 3 * B * H * npad * d * 1.1
    for bad in [(0, 1, 8, 128), (1, 0, 8, 128), (1, 1, 0, 128), (1, 1, 8, 96), (1, 70000, 8, 64)]:
        assert sage.workspace_bytes(*bad, sage.MODE_INT8_FP8) == 0
    assert sage.workspace_bytes(1, 1, 8, 128, 7) == 0


def test_argument_errors_are_host_side():
    vp = ctypes.c_void_p
    lib = sage.LIB
    fake = vp(0x100000)         # never dereferenced: validation fails first
    # bad head dim -> unsupported, before any device work
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 1, 128, 96, 0, fake, 1 << 20, None) == sage.EUNSUPPORTED
    # N = 0, null pointer, misaligned pointer, bad mode
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 1, 0, 128, 0, fake, 1 << 20, None) == sage.EINVAL
    assert lib.sage_attn_fwd(None, fake, fake, fake, 1, 1, 128, 128, 0, fake, 1 << 20, None) == sage.EINVAL
    assert lib.sage_attn_fwd(vp(0x100008), fake, fake, fake, 1, 1, 128, 128, 0, fake, 1 << 20, None) == sage.EINVAL
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 1, 128, 128, 5, fake, 1 << 20, None) == sage.EINVAL
    # workspace too small
    assert lib.sage_attn_fwd(fake, fake, fake, fake, 1, 1, 128, 128, 1, fake, 1000, None) == sage.EWORKSPACE
    # prepass with too little scratch
    assert lib.sage_quantize_qk(*([fake] * 3), 1, 1, 128, 128, *([fake] * 8), 16, None) == sage.EWORKSPACE


def test_layer_schedule_host():
    assert sage.layer_schedule(40, (0, 8, 16, 24, 32)) == [0 if l % 8 == 0 else 1 for l in range(40)]
    assert sage.layer_schedule(3, [2, 2]) == [1, 1, 0]
    with pytest.raises(sage.SageError):
        sage.layer_schedule(4, [4])
    with pytest.raises(sage.SageError):
        sage.layer_schedule(4, [-1])


def test_strerror_covers_codes():
    for c in (0, -1, -2, -3, -4, -5):
        assert sage.strerror(c) and sage.strerror(c) != "unknown status"


def test_select_full_precision_layers_host():
    import oracle
    err = [[0.01, 0.02], [0.30, 0.25], [0.05, 0.40], [0.2, 0.1]]
    # above 0.2 at every iteration: layer 1 only; means 0.015, 0.275, 0.225, 0.15
    assert sage.select_full_precision_layers(err, 0.2) == [1]
    assert sage.select_full_precision_layers(err, 0.2, sage.SELECT_MEAN) == [1, 2]
    assert sage.select_full_precision_layers(err, 0.0) == [0, 1, 2, 3]
    assert sage.select_full_precision_layers(err, 1.0) == []
    for rule in (sage.SELECT_EVERY_ITERATION, sage.SELECT_MEAN):
        for thr in (0.0, 0.05, 0.1, 0.2, 0.25, 0.3, 1.0):
            assert sage.select_full_precision_layers(err, thr, rule) == oracle.select_layers(err, thr, rule)
    with pytest.raises(sage.SageError):
        sage.select_full_precision_layers([[float("nan")]], 0.1)
    with pytest.raises(sage.SageError):
        sage.select_full_precision_layers(err, 0.1, 2)


def test_rel_l2_argument_validation_runs_on_the_host():
    lib = sage.LIB
    fake = ctypes.c_void_p(1 << 20)
    odd8 = ctypes.c_void_p((1 << 20) + 8)       # 8-byte aligned: allowed for out only
    odd4 = ctypes.c_void_p((1 << 20) + 4)
    nb = lib.sage_error_scratch_bytes(1, 2)
    assert lib.sage_attn_rel_l2(fake, fake, 1, 2, 10, 128, odd4, fake, nb, None) == sage.EINVAL
    assert lib.sage_attn_rel_l2(odd8, fake, 1, 2, 10, 128, fake, fake, nb, None) == sage.EINVAL
    assert lib.sage_attn_rel_l2(fake, fake, 1, 2, 10, 12, fake, fake, nb, None) == sage.EINVAL
    assert lib.sage_attn_rel_l2(fake, fake, 1, 2, 10, 128, fake, fake, nb - 8, None) == sage.EWORKSPACE
    assert lib.sage_attn_rel_l2(None, fake, 1, 2, 10, 128, fake, fake, nb, None) == sage.EINVAL


def test_linear_argument_validation_runs_on_the_host():
    """Bad sizes and pointers are refused before any device call (works without a GPU)."""
    lib = sage.LIB
    fake = ctypes.c_void_p(1 << 20)            # 16-byte aligned, never dereferenced on these paths
    odd = ctypes.c_void_p((1 << 20) + 4)
    s = None
    args = lambda **kw: [kw.get("xq", fake), kw.get("sx", fake), kw.get("wq", fake), kw.get("sw", fake),
                         kw.get("bias", None), kw.get("y", fake), kw.get("dt", sage.DTYPE_BF16), kw.get("M", 256),
                         kw.get("N", 256), kw.get("K", 256), kw.get("st", fake), s]
    assert lib.sage_linear_w8a8(*args(N=200)) == sage.EINVAL        # N not a multiple of 128
    assert lib.sage_linear_w8a8(*args(K=64)) == sage.EINVAL         # K below one block
    assert lib.sage_linear_w8a8(*args(M=0)) == sage.EINVAL
    assert lib.sage_linear_w8a8(*args(dt=7)) == sage.EINVAL
    assert lib.sage_linear_w8a8(*args(xq=None)) == sage.EINVAL
    assert lib.sage_linear_w8a8(*args(y=odd)) == sage.EINVAL        # misaligned output
    assert lib.sage_linear_w8a8(*args(bias=odd)) == sage.EINVAL
    assert lib.sage_dbg_linear_forced_timeout(*args()[:11], 0, s) == sage.EINVAL
    assert lib.sage_quantize_blocks_2d(fake, 100, 130, fake, fake, s) == sage.EINVAL
    assert lib.sage_quantize_blocks_2d(fake, 0, 128, fake, fake, s) == sage.EINVAL
    assert lib.sage_quantize_blocks_2d(fake, 128 * 65536, 128, fake, fake, s) == sage.EINVAL
    assert lib.sage_quantize_blocks_2d(odd, 100, 128, fake, fake, s) == sage.EINVAL
    if not _has_gpu():
        # well-formed arguments reach the device check, which reports no usable device
        assert lib.sage_linear_w8a8(*args()) in (sage.ELAUNCH, sage.EUNSUPPORTED)


def _has_gpu():
    import torch
    return torch.cuda.is_available()


def test_bf16_and_w8a16_argument_validation_runs_on_the_host():
    lib = sage.LIB
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    s = None
    assert lib.sage_linear_bf16(fake, fake, None, fake, 0, 256, 256, 96, fake, s) == sage.EINVAL   # K % 64
    assert lib.sage_linear_bf16(fake, fake, None, fake, 0, 256, 192, 128, fake, s) == sage.EINVAL  # N % 128
    assert lib.sage_linear_bf16(odd, fake, None, fake, 0, 256, 256, 128, fake, s) == sage.EINVAL
    assert lib.sage_linear_w8a16_workspace_bytes(256, 384) == 256 * 384 * 2
    assert lib.sage_linear_w8a16(fake, fake, fake, None, fake, 0, 64, 256, 192, fake, 10 ** 9, fake, s) == sage.EINVAL
    assert lib.sage_linear_w8a16(fake, fake, fake, None, fake, 0, 64, 256, 256, fake, 1000, fake, s) == sage.EWORKSPACE
    assert lib.sage_dequant_blocks_2d(fake, fake, 10, 100, fake, s) == sage.EINVAL


def test_ulysses_permute_argument_validation_runs_on_the_host():
    lib = sage.LIB
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    s = None
    assert lib.sage_ulysses_permute(a, b, 1, 10, 40, 128, 3, 0, 0, 0, s) == sage.EINVAL   # H % P
    assert lib.sage_ulysses_permute(a, b, 1, 10, 40, 96, 4, 0, 0, 0, s) == sage.EINVAL    # d
    assert lib.sage_ulysses_permute(a, b, 1, 10, 40, 128, 4, 7, 0, 0, s) == sage.EINVAL   # op
    assert lib.sage_ulysses_permute(a, a, 1, 10, 40, 128, 4, 0, 0, 0, s) == sage.EINVAL   # in place
    assert lib.sage_ulysses_permute(a, b, 1, 10, 40, 128, 4, 0, 5, 0, s) == sage.EINVAL   # chunk < dense


def test_host_chunk_rule():
    # one CTA per 256 query rows of a head; four waves of 148 SMs
    assert sage.host_chunk_heads(1, 40, 75600, 128) == 2          # 296 CTAs per head
    assert sage.host_chunk_heads(1, 30, 17776, 64) == 9           # 70 CTAs per head
    assert sage.host_chunk_heads(1, 2, 1024, 128) == 2            # capped at B*H
    assert sage.host_chunk_heads(1, 2, 1024, 96) == 0             # bad shape


def test_host_workspace_is_two_chunk_workspaces():
    """sage_attn_fwd_host keeps two chunks in flight, each with its own workspace half."""
    def one(B, H, N, d, mode, chunk):
        return (sage.workspace_bytes(1, chunk, N, d, mode) + 255) // 256 * 256
    for mode in (sage.MODE_INT8_FP8, sage.MODE_INT8_FP8_QTOKEN, sage.MODE_BF16):
        assert sage.host_workspace_bytes(1, 40, 75600, 128, mode, 0) == 2 * one(1, 40, 75600, 128, mode, 2)
        assert sage.host_workspace_bytes(2, 5, 1500, 64, mode, 3) == 2 * one(2, 5, 1500, 64, mode, 3)
        assert sage.host_workspace_bytes(1, 1, 1000, 128, mode, 0) == one(1, 1, 1000, 128, mode, 1)   # one chunk
    assert sage.host_workspace_bytes(1, 2, 1024, 96, sage.MODE_BF16, 0) == 0          # bad shape
    assert sage.host_workspace_bytes(1, 2, 1024, 128, 7, 0) == 0                      # bad mode


def test_binding_checks_what_the_c_abi_cannot_see():
    """dtype, contiguity and shape of tensor arguments are checked before any device call (CPU tensors)."""
    import torch
    xq = torch.zeros(256, 256, dtype=torch.int8)
    s = torch.zeros(2, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="int8"):
        sage.linear_w8a8(xq.float(), s, xq, s)
    with pytest.raises(ValueError, match="contiguous"):
        sage.linear_w8a8(xq.t(), s, xq, s)
    with pytest.raises(ValueError, match="shape"):
        sage.linear_w8a8(xq, torch.zeros(3, 2), xq, s)
    with pytest.raises(ValueError, match="bfloat16"):
        sage.linear_bf16(torch.zeros(4, 128), torch.zeros(128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="shape"):
        sage.linear_w8a16(torch.zeros(4, 256, dtype=torch.bfloat16), xq, s, bias=torch.zeros(3, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="shape"):
        sage.dequant_blocks_2d(xq, torch.zeros(1, 2))
    a = torch.zeros(1, 8, 4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="multiple"):
        sage.ulysses_permute(a, torch.zeros_like(a), 1, 8, 4, 16, 3, 0)
    with pytest.raises(ValueError, match=r"\[P\] side"):
        sage.ulysses_permute(a, torch.zeros(10, dtype=torch.bfloat16), 1, 8, 4, 16, 2, 0)


def test_attn_fwd_binding_checks():
    import torch
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="bfloat16"):
        sage.attn_fwd(q, q.float(), q, sage.MODE_BF16)
    with pytest.raises(ValueError, match="shape"):
        sage.attn_fwd(q, q, torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16), sage.MODE_BF16)


def test_host_tensors_are_refused_for_device_arguments():
    """The C ABI cannot tell a host address from a device one; the binding refuses CPU tensors (CPU test)."""
    import torch
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="not a CUDA tensor"):
        sage.attn_fwd(q, q, q, sage.MODE_BF16, workspace=torch.zeros(256, dtype=torch.uint8))
    x = torch.zeros(256, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="not a CUDA tensor"):
        sage.quantize_blocks_2d(x, torch.zeros(256, 256, dtype=torch.int8), torch.zeros(2, 2))
    a = torch.zeros(1, 8, 4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="not a CUDA tensor"):
        sage.ulysses_permute(a, torch.zeros_like(a), 1, 8, 4, 16, 2, 0)


def _header_decls():
    """(name, return type, [parameter types]) of every function in include/sage.h."""
    import re
    txt = re.sub(r"/\*.*?\*/", "", open(sage.HEADER).read(), flags=re.S)
    txt = re.sub(r"//[^\n]*", "", txt)
    out = []
    for m in re.finditer(r"^\s*((?:const\s+)?[A-Za-z_][\w\s\*]*?)\b([a-z_][a-z0-9_]*)\s*\(([^)]*)\)\s*;", txt, flags=re.M):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        types = [] if params in ("", "void") else [re.sub(r"\s*\b\w+$", "", p.strip()) for p in params.split(",")]
        out.append((name, ret, types))
    return out


def _ctype(c: str):
    c = " ".join(c.replace("*", " * ").split())
    if c == "const char *":
        return ctypes.c_char_p
    if "*" in c:
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "long long": ctypes.c_longlong,
            "double": ctypes.c_double}[c.replace("const ", "")]


def test_binding_signatures_match_the_header():
    """Every ctypes prototype has the header's argument count and kinds (a mismatch would pass garbage
    pointers to the device) and its return type."""
    decls = _header_decls()
    assert {n for n, _, _ in decls} == EXPECTED
    for name, ret, params in decls:
        f = getattr(sage.LIB, name)
        assert f.argtypes is not None, name
        assert [a for a in f.argtypes] == [_ctype(p) for p in params], name
        assert f.restype == _ctype(ret), name


def test_host_entry_rejects_a_workspace_off_256_bytes():
    """The host pipeline hands each half of its workspace to sage_attn_fwd (256-byte aligned); a buffer
    aligned to 16 bytes only is refused before any copy or launch (the addresses are never touched)."""
    B, H, N, d = 1, 2, 1000, 128
    p16 = ctypes.c_void_p(0x10000010)          # 16-byte aligned, not 256
    p256 = ctypes.c_void_p(0x10000100)
    n = sage.host_workspace_bytes(B, H, N, d, sage.MODE_INT8_FP8, 0)
    rc = sage.LIB.sage_attn_fwd_host(p256, p256, p256, p256, B, H, N, d, sage.MODE_INT8_FP8, p256, p256, p256, p256,
                                     p16, n, 0, None)
    assert rc == sage.EINVAL
