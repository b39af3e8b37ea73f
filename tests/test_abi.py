"""The C-ABI library loads, exports every function include/ckda.h declares,
and its host-side argument checks answer without touching a GPU."""
import ctypes

from chunked_gated_delta_ckda_b200 import _abi

P = None


def test_exports_every_header_symbol():
    lib = _abi.library()
    names = _abi.header_functions()
    assert {"ckda_chunk_fwd", "ckda_chunk_bwd", "ckda_decode_step", "ckda_varlen_fwd",
            "ckda_workspace_size", "ckda_check_device_status", "ckda_status_string",
            "ckda_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    assert _abi.ckda_status_string(0) == "ok"
    for code in range(1, 9):
        assert _abi.ckda_status_string(code) != "unknown status"
    assert _abi.ckda_version() >= 100


def test_workspace_size_rules():
    ws = _abi.ckda_workspace_size
    assert ws(0, 8, 4096, 16, 128, 128, 0) > 0
    assert ws(1, 8, 4096, 16, 128, 128, 0) > ws(0, 8, 4096, 16, 128, 128, 0)
    assert ws(2, 1, 65536, 16, 128, 128, 44) > 0
    assert ws(0, 1, 100, 2, 96, 64, 0) == 0      # unsupported dk
    assert ws(2, 2, 100, 2, 64, 64, 3) == 0      # packed call needs B == 1
    assert ws(7, 1, 100, 2, 64, 64, 0) == 0      # unknown op
    assert ws(3, 1, 65536, 16, 128, 128, 44) > ws(2, 1, 65536, 16, 128, 128, 44)  # packed backward
    assert ws(3, 2, 100, 2, 64, 64, 3) == 0      # packed backward needs B == 1
    assert ws(0, 1, 0, 2, 64, 64, 0) > 0         # empty input still has a status block


def test_saved_size_rules():
    sv = _abi.ckda_saved_size
    one = sv(1, 64, 1, 128, 128, 1)                # one (chunk, head) record
    assert one > 0 and one % 256 == 0
    assert sv(8, 4096, 16, 128, 128, 1) == 8 * 64 * 16 * one
    assert sv(2, 65, 3, 128, 128, 1) == 2 * 2 * 3 * one   # a ragged last chunk has a record
    assert sv(8, 4096, 16, 128, 128, 0) == 0       # fp32 I/O: the backward recomputes
    assert sv(8, 4096, 16, 64, 64, 1) == 0         # d = 64: the backward recomputes
    assert sv(1, 64, 2, 96, 64, 1) == 0            # unsupported dk
    assert sv(1, 0, 2, 128, 128, 1) == 0           # empty


def _raw():
    return _abi.library()


def test_host_validation_without_gpu():
    lib = _raw()
    fake = ctypes.c_void_p(1 << 20)     # never dereferenced: the calls fail validation first
    odd = ctypes.c_void_p((1 << 20) + 4)
    args = [fake] * 10
    nosave = [None, 0]

    def fwd(B, T, H, dk, dv, io, a, ws_bytes, saved=nosave):
        return lib.ckda_chunk_fwd(B, T, H, dk, dv, io, *a, *saved, fake, ws_bytes, None)

    # unsupported head size
    assert fwd(1, 64, 2, 96, 64, 0, args, 1 << 30) == 2
    # bad io dtype
    assert fwd(1, 64, 2, 64, 64, 5, args, 1 << 30) == 1
    # negative sizes
    assert fwd(-1, 64, 2, 64, 64, 0, args, 1 << 30) == 1
    # null required pointer
    a = list(args)
    a[0] = None
    assert fwd(1, 64, 2, 64, 64, 0, a, 1 << 30) == 1
    # misaligned tensor
    a = list(args)
    a[1] = odd
    assert fwd(1, 64, 2, 64, 64, 0, a, 1 << 30) == 3
    # workspace too small
    assert fwd(1, 64, 2, 64, 64, 0, args, 16) == 4
    # sequences and heads index grid dimensions: at most 65535 each
    assert fwd(70000, 1, 2, 64, 64, 0, args, 1 << 30) == 2
    assert fwd(1, 64, 70000, 64, 64, 0, args, 1 << 30) == 2
    assert lib.ckda_workspace_size(0, 70000, 1, 2, 64, 64, 0) == 0
    assert lib.ckda_workspace_size(2, 1, 100000, 2, 64, 64, 70000) == 0
    # saved buffer: too small / misaligned where the configuration has a saved form
    need = lib.ckda_saved_size(1, 64, 2, 128, 128, 1)
    assert fwd(1, 64, 2, 128, 128, 1, args, 1 << 30, [fake, need - 1]) == 4
    assert fwd(1, 64, 2, 128, 128, 1, args, 1 << 30, [ctypes.c_void_p((1 << 20) + 16), need]) == 3
    # decode: unsupported / null
    assert lib.ckda_decode_step(4, 2, 64, 32, 0, *([fake] * 8), None) == 2
    assert lib.ckda_decode_step(4, 2, 64, 64, 0, *([None] * 8), None) == 1
    # packed: bad max_seqlen, N < 0
    v = [fake] * 9
    assert lib.ckda_varlen_fwd(100, 2, fake, 0, 2, 64, 64, 0, *v, None, 0, fake, 1 << 30, None) == 1
    assert lib.ckda_varlen_fwd(100, -1, fake, 50, 2, 64, 64, 0, *v, None, 0, fake, 1 << 30, None) == 1
    assert lib.ckda_varlen_fwd(100000, 70000, fake, 50, 2, 64, 64, 0, *v, None, 0, fake, 1 << 30, None) == 2
    need = lib.ckda_varlen_saved_size(100, 2, 2, 128, 128, 1)
    assert need > 0 and lib.ckda_varlen_saved_size(100, 2, 2, 64, 64, 0) == 0
    assert lib.ckda_varlen_fwd(100, 2, fake, 50, 2, 128, 128, 1, *v, fake, need - 1, fake, 1 << 30, None) == 4
    vb = [fake] * 9 + [None, 0] + [fake] * 6
    assert lib.ckda_varlen_bwd(100, 2, fake, 0, 2, 64, 64, 0, *vb, fake, 1 << 30, None) == 1   # max_seqlen
    assert lib.ckda_varlen_bwd(100, 2, None, 50, 2, 64, 64, 0, *vb, fake, 1 << 30, None) == 1  # cu_seqlens
    assert lib.ckda_varlen_bwd(100, 2, fake, 50, 2, 64, 64, 0, *vb, fake, 16, None) == 4       # workspace
    assert lib.ckda_varlen_bwd(0, 0, fake, 0, 2, 64, 64, 0, *vb, fake, 1 << 30, None) == 0     # nothing to do

    def bwd(io, b, ws_bytes, saved=nosave):
        return lib.ckda_chunk_bwd(1, 64, 2, 128, 128, io, *b[:10], *saved, *b[10:], fake, ws_bytes, None)

    # backward: missing gradient output
    b = [fake] * 16
    b[13] = None  # dg
    assert bwd(1, b, 1 << 30) == 1
    # backward: workspace too small
    b[13] = fake
    assert bwd(1, b, 16) == 4
    # backward: saved buffer too small (bf16, d = 128 has a saved form)
    assert bwd(1, b, 1 << 30, [fake, 16]) == 4
    # zero-sized decode is a no-op
    assert lib.ckda_decode_step(0, 2, 64, 64, 0, *([None] * 8), None) == 0

    def multi(N=4, K=3, dk=64, dv=64, io=0, ptrs=None, n_tokens=None, slots=None, n_slots=4, write=1):
        p = [fake] * 6 if ptrs is None else ptrs
        return lib.ckda_decode_multi(N, K, 2, dk, dv, io, *p, n_tokens, slots, n_slots, fake, write, fake, None)

    assert multi(N=-1) == 1 and multi(K=-1) == 1
    assert multi(dk=96) == 2
    assert multi(io=7) == 1
    assert multi(write=2) == 1
    assert multi(n_slots=3) == 1                      # identity slots need n_slots >= N
    assert multi(n_slots=-1, slots=fake) == 1
    assert multi(ptrs=[None] + [fake] * 5) == 1       # q missing
    assert multi(ptrs=[fake, odd] + [fake] * 4) == 3  # k misaligned
    assert multi(n_tokens=ctypes.c_void_p((1 << 20) + 2)) == 3
    assert multi(N=0) == 0 and multi(K=0) == 0        # nothing to do
    assert multi(N=1 << 29, K=1, n_slots=1 << 29) == 2  # grid: N * H CTAs
    # failure-detection self-test: workspace checks come before the launch
    assert lib.ckda_selftest_bounded_wait(None, 256, 1, None) == 1
    assert lib.ckda_selftest_bounded_wait(fake, 255, 1, None) == 4
    assert lib.ckda_selftest_bounded_wait(ctypes.c_void_p((1 << 20) + 16), 256, 1, None) == 3
    assert lib.ckda_decode_step(1 << 29, 4, 64, 64, 0, *([fake] * 8), None) == 2

    F = ctypes.c_float
    pf = lambda B=1, T=8, dk=64, io=0, floor=-5.0, ptrs=None, cu=None, n=0: lib.ckda_prologue_fwd(
        B, T, 2, dk, 64, io, *([fake] * 8 if ptrs is None else ptrs), F(floor), cu, n, *([fake] * 6), None)
    assert pf(B=-1) == 1 and pf(io=3) == 1 and pf(dk=32) == 2
    assert pf(floor=0.5) == 1 and pf(floor=float("-inf")) == 1 and pf(floor=float("nan")) == 1
    assert pf(B=70000) == 2                          # grid limit on B and H
    assert pf(ptrs=[fake] * 7 + [None]) == 1         # b missing
    assert pf(ptrs=[odd] + [fake] * 7) == 3
    assert pf(T=0) == 0                              # empty: nothing to do
    assert pf(B=2, cu=fake, n=2) == 1                # packed documents take one row
    assert pf(cu=fake, n=0) == 1                     # ... and at least one document
    assert pf(cu=ctypes.c_void_p((1 << 20) + 2), n=2) == 3
    pb = lambda dw=fake, floor=-5.0, B=1, cu=None, n=0: lib.ckda_prologue_bwd(
        B, 8, 2, 64, 64, 0, *([fake] * 8), F(floor), cu, n, *([fake] * 5), fake, fake, fake, dw, fake, fake, fake,
        fake, None)
    assert pb(dw=None) == 1 and pb(floor=1.0) == 1
    assert pb(B=2, cu=fake, n=1) == 1 and pb(cu=fake, n=-1) == 1
