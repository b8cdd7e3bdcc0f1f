"""The C-ABI library loads on a machine without a GPU and exports every symbol gqa.h declares;
host-side argument checks run before any CUDA call. No compute is launched here."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\**\s+\**([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


@pytest.fixture(scope="module")
def lib():
    from kv_cache_attention_gqa_b200 import _lib

    return _lib._lib


def test_header_declares_the_three_entry_points():
    names = _declared_functions()
    for n in ("gqa_prefill", "gqa_decode", "kv_append", "gqa_decode_workspace_size",
              "gqa_get_device_error", "gqa_status_string", "gqa_version"):
        assert n in names, names


def test_library_exports_every_declared_symbol(lib):
    from kv_cache_attention_gqa_b200 import _lib

    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in _declared_functions():
        assert n in exported, f"{n} not exported"
        assert hasattr(lib, n)
    assert set(_lib.SIGNATURES) == set(_declared_functions())


def test_status_strings_and_version(lib):
    from kv_cache_attention_gqa_b200 import _lib

    for code, name in _lib.STATUS_NAMES.items():
        assert lib.gqa_status_string(code).decode() == name
    assert b"sm_100a" in lib.gqa_version()


def test_expire_waits_hook_takes_only_zero_or_one(lib):
    assert lib.gqa_debug_expire_waits(2) == 1
    assert lib.gqa_debug_expire_waits(-1) == 1
    assert lib.gqa_debug_expire_waits(1) == 0
    assert lib.gqa_debug_expire_waits(0) == 0  # left off


def test_host_side_argument_errors(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)
    null = None
    s = None
    # null pointers
    assert lib.gqa_prefill(null, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, 0.125, 1, 0, 0, s) == 1
    # h_q not a multiple of h_kv
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 6, 4, 8, 8, 64, 0.125, 1, 0, 0, s) == 1
    # non-positive sizes, bad scale, bad causal flag
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 0, 4, 2, 8, 8, 64, 0.125, 1, 0, 0, s) == 1
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, float("nan"), 1, 0, 0, s) == 1
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, -1.0, 1, 0, 0, s) == 1
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, 0.1, 2, 0, 0, s) == 1
    # sliding window: negative, or without the causal mask
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, 0.1, 1, -1, 0, s) == 1
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, 0.1, 0, 4, 0, s) == 1
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, -1, 0, fake, 1 << 20, 1, s) == 1
    # prefill: unsupported head dims, an unknown dtype and sizes past 32-bit row indexing, all reported
    # before any CUDA call
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 96, 0.1, 1, 0, 0, s) == 2
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 300, 0.1, 1, 0, 1, s) == 2
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, 0.1, 1, 0, 7, s) == 1
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1024, 32, 32, 8, 65536, 128, 0.1, 1, 0, 0, s) == 2
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1024, 32, 8, 65536, 8, 128, 0.1, 1, 0, 0, s) == 2
    # decode: cache rows past 32-bit row indexing
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1024, 32, 32, 65536, 128, 0.1, 0, 0, fake,
                          1 << 20, 1, s) == 2
    assert lib.gqa_decode_noalloc(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, -1, 0, 1, s) == 1
    # the no-alloc decode applies gqa_decode's checks first: a batch beyond the decode limit and a bf16
    # d_h outside {64, 128} are UNSUPPORTED (not WORKSPACE, though their workspace would also exceed the
    # fixed scratch array); a null output is INVALID_ARG
    assert lib.gqa_decode_noalloc(fake, fake, fake, fake, null, null, null, 2000, 64, 64, 4096, 128, 0.1, 0, 0,
                                  100000, s) == 2
    assert lib.gqa_decode_noalloc(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 96, 0.1, 0, 0, 1, s) == 2
    assert lib.gqa_decode_noalloc(fake, fake, fake, null, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, 1, s) == 1
    # scale: 0 selects the default 1/sqrt(d_h); negative, NaN and infinite scales are refused
    for bad in (-0.5, float("nan"), float("inf"), float("-inf")):
        assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 64, bad, 1, 0, 0, s) == 1
        assert lib.gqa_decode_noalloc(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, bad, 0, 0, 1, s) == 1
    # scale 0 passes the host checks (the next refusal is the unsupported d_h)
    assert lib.gqa_prefill(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 8, 96, 0.0, 1, 0, 0, s) == 2
    # decode
    assert lib.gqa_decode(null, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, fake, 1 << 20, 1, s) == 1
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 3, 8, 64, 0.1, 0, 0, fake, 1 << 20, 1, s) == 1
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, fake, 1 << 20, -1, s) == 1
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 7, fake, 1 << 20, 1, s) == 1
    # unsupported: bf16 with d_h = 96; batch beyond the decode limit
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 96, 0.1, 0, 0, fake, 1 << 20, 1, s) == 2
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 5000, 4, 2, 8, 64, 0.1, 0, 0, fake, 1 << 20, 1, s) == 2
    # workspace: missing, too small, misaligned (num_splits given, so no device query is needed)
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, null, 1 << 20, 1, s) == 5
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, fake, 16, 1, s) == 5
    assert lib.gqa_decode(fake, fake, fake, fake, null, null, null, 1, 4, 2, 8, 64, 0.1, 0, 0, P(0x1004), 1 << 20, 1, s) == 5
    # kv_append
    assert lib.kv_append(fake, fake, fake, fake, null, 1, 2, 1, 8, 64, 0, s) == 1
    assert lib.kv_append(null, fake, fake, fake, fake, 1, 2, 1, 8, 64, 0, s) == 1
    assert lib.kv_append(fake, fake, null, null, null, 1, 2, 0, 8, 64, 0, s) == 0  # zero rows: no-op
    assert lib.kv_append(fake, fake, fake, fake, fake, 1, 2, 9, 8, 64, 0, s) == 1
    assert lib.kv_append(fake, fake, fake, fake, fake, 1, 2, 1, 8, 64, 9, s) == 1
    assert lib.gqa_get_device_error(None, s) == 1


def test_workspace_size(lib):
    assert lib.gqa_decode_workspace_size(1, 6, 4, 8, 64, 0, 4) == 0
    assert lib.gqa_decode_workspace_size(0, 4, 2, 8, 64, 0, 4) == 0
    a = lib.gqa_decode_workspace_size(8, 32, 8, 8192, 128, 0, 148)
    b = lib.gqa_decode_workspace_size(8, 32, 8, 8192, 128, 0, 296)
    assert 0 < a < b
    # partials: (splits + units) slots of r heads x (d_h + 1) floats, plus one counter per unit
    assert a >= (148 + 64) * 4 * 129 * 4 + 64 * 4


def test_mla_workspace_size_follows_the_kernel_the_call_selects(lib):
    """With explicit splits the size needs no device. bf16 with a multiple of 128 heads runs the
    tensor-core kernel (units of 128 heads, one partial row per head of a unit); fp32 and other
    head counts run 16-head units. Layout: a 256-byte header, the prefix sums and lengths of the
    sequences, then (splits + units) partial slots of lse and of d_v floats per unit head, each
    region 256-byte aligned."""
    def expected(B, units, hpu, d_v, splits):
        al = lambda x: (x + 255) // 256 * 256  # noqa: E731
        slots = splits + units
        return 256 + al((B + 1) * 8) + al(B * 4) + al(slots * hpu * 4) + slots * hpu * d_v * 4

    bf16, fp32 = 0, 1
    assert lib.gqa_mla_decode_workspace_size(8, 128, 8192, 512, bf16, 200) == expected(8, 8, 128, 512, 200)
    assert lib.gqa_mla_decode_workspace_size(8, 256, 8192, 512, bf16, 7) == expected(8, 16, 128, 512, 7)
    assert lib.gqa_mla_decode_workspace_size(8, 16, 8192, 512, bf16, 7) == expected(8, 8, 16, 512, 7)
    assert lib.gqa_mla_decode_workspace_size(8, 128, 8192, 512, fp32, 7) == expected(8, 64, 16, 512, 7)


def test_paged_host_side_argument_errors(lib):
    """gqa_decode_paged / kv_append_paged reject bad page geometry before any CUDA call."""
    P = ctypes.c_void_p
    fake = P(0x1000)
    null = None
    s = None
    # args: q, k_pages, v_pages, o, lse, kv_len, q_pos, block_table,
    #       B, h_q, h_kv, num_pages, page_size, max_pages, d_h, scale, window, dtype, ws, ws_bytes,
    #       splits, stream
    ok = [fake, fake, fake, fake, null, null, null, fake, 1, 4, 2, 8, 16, 4, 64, 0.1, 0, 0, fake, 1 << 20, 1, s]

    def dec(**kw):
        a = list(ok)
        idx = {"bt": 7, "num_pages": 11, "page_size": 12, "max_pages": 13, "d_h": 14, "window": 16, "ws": 18}
        for k, v in kw.items():
            a[idx[k]] = v
        return lib.gqa_decode_paged(*a)

    assert dec(bt=null) == 1
    assert dec(num_pages=0) == 1
    assert dec(page_size=0) == 1
    assert dec(max_pages=0) == 1
    assert dec(page_size=24) == 2          # not a multiple of 16
    assert dec(d_h=96) == 2                # bf16 head dims are 64 / 128
    assert dec(page_size=1 << 16, max_pages=1 << 16) == 2  # T_max beyond 2^31
    assert dec(page_size=1 << 12, num_pages=1 << 18) == 2  # pool rows beyond 2^31
    assert dec(ws=null) == 5
    assert dec(window=-1) == 1
    # kv_append_paged: k, v, k_new, v_new, pos, block_table, B, h_kv, S_new, num_pages, page_size,
    #                  max_pages, d_h, dtype, stream
    assert lib.kv_append_paged(fake, fake, fake, fake, fake, null, 1, 2, 1, 8, 16, 4, 64, 0, s) == 1
    assert lib.kv_append_paged(fake, fake, null, null, null, null, 1, 2, 0, 8, 16, 4, 64, 0, s) == 0
    assert lib.kv_append_paged(fake, fake, fake, fake, null, fake, 1, 2, 1, 8, 16, 4, 64, 0, s) == 1
    assert lib.kv_append_paged(fake, fake, fake, fake, fake, fake, 1, 2, 1, 0, 16, 4, 64, 0, s) == 1
    assert lib.kv_append_paged(fake, fake, fake, fake, fake, fake, 1, 2, 65, 8, 16, 4, 64, 0, s) == 1
    assert lib.kv_append_paged(fake, fake, fake, fake, fake, fake, 1, 2, 1, 8, 16, 4, 64, 7, s) == 1


def test_mla_and_backward_host_side_argument_errors(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)
    null = None
    s = None
    # gqa_mla_decode(q, cache, o, lse, kv_len, q_pos, B, h_q, T_max, d_qk, d_v, scale, dtype, ws, bytes, splits, stream)
    mla = lambda *a: lib.gqa_mla_decode(*a)  # noqa: E731
    assert mla(null, fake, fake, null, null, null, 2, 16, 64, 576, 512, 0.07, 0, fake, 1 << 20, 1, s) == 1
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 512, 576, 0.07, 0, fake, 1 << 20, 1, s) == 1  # d_v > d_qk
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 576, 512, -1.0, 0, fake, 1 << 20, 1, s) == 1
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 576, 256, 0.07, 0, fake, 1 << 20, 1, s) == 2  # bf16 widths
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 800, 512, 0.07, 1, fake, 1 << 20, 1, s) == 2  # fp32 limit
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 576, 512, 0.07, 0, null, 1 << 20, 1, s) == 5
    assert mla(fake, fake, fake, null, null, null, 2, 16, 64, 576, 512, 0.07, 0, fake, 16, 1, s) == 5
    assert lib.gqa_mla_decode_workspace_size(0, 16, 64, 512, 0, 1) == 0
    assert lib.gqa_mla_decode_workspace_size(2, 16, 64, 512, 0, 4) > 0
    # gqa_prefill_backward(q, k, v, o, dO, lse, dq, dk, dv, q_start, kv_len, B, h_q, h_kv, S_q, T_max, d_h,
    #                      scale, causal, window, dtype, ws, bytes, stream)
    ok = [fake] * 9 + [null, null, 1, 4, 2, 8, 8, 64, 0.125, 1, 0, 0, fake, 1 << 20, s]

    def bwd(**kw):
        a = list(ok)
        idx = {"lse": 5, "dq": 6, "h_kv": 13, "d_h": 16, "causal": 18, "window": 19, "ws": 21, "bytes": 22}
        for k, v in kw.items():
            a[idx[k]] = v
        return lib.gqa_prefill_backward(*a)

    assert bwd(lse=null) == 1
    assert bwd(dq=null) == 1
    assert bwd(h_kv=3) == 1
    assert bwd(causal=0, window=4) == 1
    assert bwd(window=-2) == 1
    assert bwd(d_h=96) == 2
    assert bwd(ws=null) == 5
    assert bwd(ws=P(0x1010)) == 5  # misaligned
    assert bwd(bytes=8) == 5
    assert lib.gqa_prefill_backward_workspace_size(1, 4, 8) == 3 * 256  # lse2, D, item counter
    assert lib.gqa_prefill_backward_workspace_size(0, 4, 8) == 0


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on a machine without a GPU (only what the binding's checks read)."""

    def __init__(self, index, contiguous=True):
        import torch

        self.is_cuda = True
        self.device = torch.device("cuda", index)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous


def test_binding_rejects_tensors_off_the_current_device(monkeypatch):
    """The library launches on the current device and stream, so every tensor must live there."""
    import torch

    from kv_cache_attention_gqa_b200 import _lib

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    _lib._need_cuda(_FakeCudaTensor(1), None, _FakeCudaTensor(1))
    with pytest.raises(ValueError, match="current CUDA device"):
        _lib._need_cuda(_FakeCudaTensor(1), _FakeCudaTensor(0))
    with pytest.raises(ValueError, match="contiguous"):
        _lib._need_cuda(_FakeCudaTensor(1, contiguous=False))
    with pytest.raises(ValueError, match="CUDA device"):
        _lib._need_cuda(torch.zeros(2))


def test_binding_checks_caller_outputs_and_workspaces(monkeypatch):
    """A caller's output must have the exact shape and dtype the kernel writes; a caller's
    workspace is sized in bytes whatever its element type, and must be a device tensor."""
    import torch

    from kv_cache_attention_gqa_b200 import _lib

    out = torch.empty(2, 3, 4, dtype=torch.bfloat16)
    assert _lib._out(out, (2, 3, 4), torch.bfloat16, "cpu") is out
    assert _lib._out(None, (2, 3, 4), torch.float32, "cpu").shape == (2, 3, 4)
    with pytest.raises(ValueError, match="shape"):
        _lib._out(out, (2, 3, 5), torch.bfloat16, "cpu")
    with pytest.raises(ValueError, match="shape"):
        _lib._out(out, (2, 3, 4), torch.float32, "cpu")
    with pytest.raises(ValueError, match="CUDA device"):
        _lib._ws_bytes(torch.zeros(16, dtype=torch.uint8))

    class _FakeWs(_FakeCudaTensor):
        def numel(self):
            return 10

        def element_size(self):
            return 4

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert _lib._ws_bytes(_FakeWs(0)) == 40


def test_plain_c_client_compiles_links_and_runs(tmp_path):
    """gqa.h is a C header (strict C99, no C++ or CUDA types in the signatures): a C program that
    includes only it links against the library and makes the host-only calls."""
    import shutil

    from kv_cache_attention_gqa_b200 import _lib

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "client")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_client.c"), "-o", exe, "-L", lib_dir, "-lgqa_b200",
                    "-Wl,-rpath," + lib_dir], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "sm_100a" in r.stdout
