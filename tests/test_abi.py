"""The C-ABI library loads without a GPU, exports every entry point include/gdn.h declares,
and rejects bad arguments on the host before any launch (these calls compute nothing)."""
import ctypes
import os
import re

import pytest

from gated_deltanet_mixer_verify_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def gdn():
    gbuild.build()
    from gated_deltanet_mixer_verify_b200 import gdn as g
    return g


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(gdn):
    names = declared_functions()
    assert {"gdn_verify_step", "gdn_commit", "gdn_decode_step", "gdn_chunk_prefill"} <= set(names)
    lib = gdn.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(gdn):
    lib = gdn.lib()
    assert lib.gdn_abi_version() == 10
    for code in (0, -1, -2, -3, -4):
        assert lib.gdn_status_string(code).decode().startswith("GDN_")
    assert "unknown" in lib.gdn_status_string(7).decode()


def test_stash_bytes_formula(gdn):
    # khat [T][d_k] + G [T pad 4] + u [T*d_v pad 4] floats per (sequence, value head)
    def per_head(T, dk, dv):
        pad = lambda x: (x + 3) // 4 * 4
        return T * dk + pad(T) + pad(T * dv)
    assert gdn.stash_bytes(64, 8, 16, 48, 128, 128) == 64 * 48 * per_head(8, 128, 128) * 4
    assert gdn.stash_bytes(1, 3, 1, 1, 16, 5) == per_head(3, 16, 5) * 4
    assert gdn.stash_bytes(1, 17, 1, 1, 16, 16) == 0          # T > 16: not a verify shape


def _call_verify(gdn, shape, ptrs=None, accept=True):
    p = ptrs or {}
    fake = 0x10000
    get = lambda k: p.get(k, fake)
    return gdn.lib().gdn_verify_step(
        ctypes.byref(shape) if shape is not None else None, get("q"), get("k"), get("v"), get("a"),
        get("b"), get("A_log"), get("dt_bias"), get("state_in"), get("state_out"),
        get("accept_len") if accept else None, get("o"), p.get("stash"), None)


def test_host_validation_rejects_before_launch(gdn):
    INVALID, UNSUP = -1, -2
    ok_shape = lambda **kw: gdn.make_shape(**dict(dict(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128), **kw))
    assert _call_verify(gdn, None) == INVALID
    assert _call_verify(gdn, ok_shape(H_v=47)) == INVALID             # H_v % H_k
    assert _call_verify(gdn, ok_shape(T=0)) == INVALID
    assert _call_verify(gdn, ok_shape(B=-1)) == INVALID
    assert _call_verify(gdn, ok_shape(d_k=96)) == UNSUP
    assert _call_verify(gdn, ok_shape(T=17)) == UNSUP
    assert _call_verify(gdn, ok_shape(), {"q": None}) == INVALID      # NULL tensor
    assert "q is NULL" in gdn.lib().gdn_last_error().decode()
    assert _call_verify(gdn, ok_shape(), {"v": 0x10008}) == INVALID   # misaligned
    assert "not 16-byte aligned" in gdn.lib().gdn_last_error().decode()
    # two-phase without a stash
    assert _call_verify(gdn, ok_shape(), accept=False) == INVALID
    # partial overlap of state_out with state_in
    assert _call_verify(gdn, ok_shape(), {"state_in": 0x100000, "state_out": 0x100010}) == INVALID
    # decode needs T == 1
    lib = gdn.lib()
    sh = ok_shape(T=2)
    assert lib.gdn_decode_step(ctypes.byref(sh), *([0x10000] * 9), None) == UNSUP
    # prefill: only chunk 64 with d = 128 is built; workspace checked
    sh = ok_shape(T=4096)
    assert lib.gdn_chunk_prefill(ctypes.byref(sh), 32, *([0x10000] * 11), 0, None) == UNSUP
    sh = ok_shape(T=4096, d_k=64, d_v=64)
    assert lib.gdn_chunk_prefill(ctypes.byref(sh), 64, *([0x10000] * 11), 0, None) == UNSUP
    # the no-allocation prefill refuses shapes larger than its fixed scratch, before any launch
    sh = ok_shape(B=1, T=4096)
    assert lib.gdn_chunk_prefill_noalloc(ctypes.byref(sh), 64, *([0x10000] * 10), None) == UNSUP
    assert "fixed scratch" in lib.gdn_last_error().decode()


def test_empty_batch_is_a_no_op(gdn):
    sh = gdn.make_shape(B=0, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    assert gdn.lib().gdn_verify_step(ctypes.byref(sh), *([None] * 12), None) == 0
    assert gdn.lib().gdn_commit(ctypes.byref(sh), None, None, None, None, None) == 0


def test_prefill_phase_entry_points_validate_on_the_host(gdn):
    INVALID, UNSUP, WORKSPACE = -1, -2, -4
    lib = gdn.lib()
    sh = gdn.make_shape(B=1, T=300, H_k=2, H_v=6, d_k=128, d_v=128)
    need = gdn.prefill_workspace_bytes(1, 300, 2, 6, 128, 128)
    # 5 chunks: 2 key heads x 65,536 + 6 value heads x 49,728 bytes per chunk
    assert need == 5 * (2 * 65536 + 6 * 49728)
    fake = 0x10000
    prep = lambda chunk, ws, nbytes, **kw: lib.gdn_chunk_prefill_prepare(
        ctypes.byref(sh), chunk, kw.get("q", fake), fake, fake, fake, fake, fake, ws, nbytes, None)
    scan = lambda chunk, ws, nbytes, **kw: lib.gdn_chunk_prefill_scan(
        ctypes.byref(sh), chunk, kw.get("v", fake), None, fake, fake, ws, nbytes, None)
    assert prep(64, None, 0) == WORKSPACE
    assert scan(64, fake, need - 16) == WORKSPACE
    assert "workspace of %d bytes needed" % need in lib.gdn_last_error().decode()
    assert prep(32, fake, need) == UNSUP
    assert scan(64, fake + 8, need) == INVALID                     # misaligned workspace
    assert prep(64, fake, need, q=None) == INVALID
    assert "q is NULL" in lib.gdn_last_error().decode()
    assert scan(64, fake, need, v=None) == INVALID
    assert "v is NULL" in lib.gdn_last_error().decode()
    empty = gdn.make_shape(B=0, T=300, H_k=2, H_v=6, d_k=128, d_v=128)
    assert lib.gdn_chunk_prefill_scan(ctypes.byref(empty), 64, *([None] * 5), 0, None) == 0


def test_prefill_piece_rule(gdn):
    # n = ceil(T / 64) chunks: min(4, max(1, n / 32)) pieces; 0 for an empty prompt
    for T, want in ((0, 0), (1, 1), (2048, 1), (4032, 1), (4033, 2), (4096, 2), (6144, 3),
                    (8128, 3), (8129, 4), (8192, 4), (8197, 4), (32768, 4), (1 << 24, 4)):
        assert gdn.chunk_prefill_pieces(T) == want, T
    assert gdn.chunk_prefill_pieces(-1) == -1
    assert gdn.chunk_prefill_pieces(4096, chunk=32) == -1


def test_commit_and_verify_validates_on_the_host(gdn):
    INVALID, UNSUP = -1, -2
    lib = gdn.lib()
    fake = 0x10000
    sh = gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    call = lambda prev_T, **kw: lib.gdn_commit_and_verify(
        ctypes.byref(kw.get("shape", sh)), prev_T, *([fake] * 7), kw.get("state", fake), kw.get("prev_stash", fake),
        kw.get("prev_L", fake), kw.get("L", fake), fake, kw.get("stash", fake), None)
    assert call(0) == INVALID and "prev_T" in lib.gdn_last_error().decode()
    assert call(17) == INVALID
    assert call(8, prev_stash=None) == INVALID and "prev_stash is NULL" in lib.gdn_last_error().decode()
    assert call(8, prev_L=None) == INVALID
    assert call(8, state=None) == INVALID
    assert call(8, L=None, stash=None) == INVALID and "stash is required" in lib.gdn_last_error().decode()
    assert call(8, shape=gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=96, d_v=128)) == UNSUP
    empty = gdn.make_shape(B=0, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    assert lib.gdn_commit_and_verify(ctypes.byref(empty), 8, *([None] * 13), None) == 0


def test_short_conv_validates_on_the_host(gdn):
    INVALID, UNSUP = -1, -2
    lib = gdn.lib()
    fake = 0x100000
    sh = gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    C = gdn.conv_channels(16, 48, 128, 128)
    assert C == 10240
    hist_bytes = 2 * 3 * C * 2
    call = lambda K=4, **kw: lib.gdn_short_conv(
        ctypes.byref(kw.get("shape", sh)), K, kw.get("q", fake), fake, fake, kw.get("w", fake), kw.get("h", fake),
        kw.get("ho", fake), None, kw.get("qo", 0x4000000), kw.get("ko", 0x5000000), kw.get("vo", 0x6000000), None)
    assert call(K=5) == UNSUP and "conv_k" in lib.gdn_last_error().decode()
    assert call(K=1) == UNSUP
    assert call(shape=gdn.make_shape(B=2, T=8, H_k=1, H_v=1, d_k=16, d_v=12)) == UNSUP
    assert call(ko=None) == INVALID and "all given or all NULL" in lib.gdn_last_error().decode()
    assert call(qo=None, ko=None, vo=None, ho=None) == INVALID and "nothing to write" in lib.gdn_last_error().decode()
    assert call(q=None) == INVALID and "q is NULL" in lib.gdn_last_error().decode()
    assert call(w=None) == INVALID and "conv_w is NULL" in lib.gdn_last_error().decode()
    assert call(h=fake + 8) == INVALID and "not 16-byte aligned" in lib.gdn_last_error().decode()
    assert call(ho=fake + 16) == INVALID and "partially overlaps" in lib.gdn_last_error().decode()
    assert call(qo=fake) == INVALID and "overlaps" in lib.gdn_last_error().decode()       # output on an input
    assert call(vo=fake + hist_bytes - 16, h=fake + 0x2000000, ho=fake + hist_bytes - 32 + 0x2000000) == INVALID
    # rewind only: no weights needed
    empty = gdn.make_shape(B=0, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    assert lib.gdn_short_conv(ctypes.byref(empty), 4, *([None] * 6), None, None, None, None, None) == INVALID
    assert lib.gdn_short_conv(ctypes.byref(empty), 4, *([None] * 5), fake, None, None, None, None, None) == 0


def test_gated_norm_entry_points_validate_on_the_host(gdn):
    INVALID, UNSUP = -1, -2
    lib = gdn.lib()
    fake = 0x100000
    F32, BF16 = 0, 1
    norm = lambda rows=4, d=128, x=fake, y=0x200000, xt=F32, yt=F32, eps=1e-6: lib.gdn_gated_rmsnorm(
        rows, d, x, xt, fake, BF16, fake, eps, y, yt, None)
    assert norm(d=126) == INVALID and "multiple of 4" in lib.gdn_last_error().decode()
    assert norm(d=8192) == INVALID
    assert norm(eps=-1.0) == INVALID
    assert norm(xt=7) == INVALID and "dtype 7" in lib.gdn_last_error().decode()
    assert norm(y=fake + 16) == INVALID and "partially overlaps" in lib.gdn_last_error().decode()
    assert norm(y=fake, yt=BF16) == INVALID and "one dtype" in lib.gdn_last_error().decode()
    assert norm(x=fake + 8) == INVALID and "not 16-byte aligned" in lib.gdn_last_error().decode()
    assert norm(rows=0, x=None, y=None) == 0
    sh = gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128)
    gated = lambda z=fake, w=fake, eps=1e-6, shape=sh: lib.gdn_verify_step_gated(
        ctypes.byref(shape), *([fake] * 8), None, fake, z, w, eps, fake, None, None)
    assert gated(z=None) == INVALID and "norm_z is NULL" in lib.gdn_last_error().decode()
    assert gated(w=None) == INVALID and "norm_w is NULL" in lib.gdn_last_error().decode()
    assert gated(eps=-1.0) == INVALID
    assert gated(shape=gdn.make_shape(B=2, T=8, H_k=1, H_v=1, d_k=16, d_v=18)) == UNSUP


def test_accept_validates_on_the_host(gdn):
    INVALID, UNSUP, WORKSPACE = -1, -2, -4
    lib = gdn.lib()
    fake = 0x100000
    need = gdn.accept_workspace_bytes(64, 8, 151936, True)
    # row statistics (16 bytes a row: 8 target + 7 draft rows per sequence), two counters, a
    # flag and n per sequence, tile sums (594 tiles of 256 logits)
    assert need == 64 * 15 * 16 + 3 * 64 * 4 + 64 * 4 + 64 * 594 * 4 + 64
    assert gdn.accept_workspace_bytes(64, 8, 151936, False) == 64 * 8 * 16 + 3 * 64 * 4 + 64 * 4 + 64
    assert gdn.accept_workspace_bytes(1, 8, (1 << 18) + 8, True) == 0
    call = lambda V=1024, T=8, sampled=1, tau=1.0, ws=fake, nbytes=1 << 30, draft=fake, u=fake, dtype=1: lib.gdn_accept(
        ctypes.byref(gdn._accept_shape(4, T, V, gdn.torch.bfloat16 if dtype else gdn.torch.float32, sampled, tau)),
        fake, draft, fake, u, fake, fake, ws, nbytes, None)
    assert call(V=1020) == UNSUP and "multiple of 8" in lib.gdn_last_error().decode()
    assert call(T=17) == UNSUP
    assert call(tau=0.0) == INVALID and "temperature" in lib.gdn_last_error().decode()
    assert call(draft=None) == INVALID and "draft_logits is NULL" in lib.gdn_last_error().decode()
    assert call(u=None) == INVALID and "uniforms is NULL" in lib.gdn_last_error().decode()
    assert call(sampled=0, draft=None, u=None, nbytes=16) == WORKSPACE
    assert call(ws=fake + 8) == INVALID and "workspace not 16-byte aligned" in lib.gdn_last_error().decode()


def test_selftest_bounded_wait_validates_on_the_host(gdn):
    lib = gdn.lib()
    assert lib.gdn_selftest_bounded_wait(None, 16, None) == -1
    assert lib.gdn_selftest_bounded_wait(0x100002, 16, None) == -1          # misaligned
    assert lib.gdn_selftest_bounded_wait(0x100000, 0, None) == -1
    assert lib.gdn_selftest_bounded_wait(0x100000, (1 << 20) + 1, None) == -1


def test_package_exports_every_binding_entry_point(gdn):
    import gated_deltanet_mixer_verify_b200 as pkg
    public = {n for n, v in vars(gdn).items()
              if not n.startswith("_") and callable(v) and getattr(v, "__module__", None) == gdn.__name__}
    assert public <= set(pkg.__all__), sorted(public - set(pkg.__all__))
    for n in pkg.__all__:
        assert getattr(pkg, n) is getattr(gdn, n), n


def test_binding_rejects_element_types_the_abi_does_not_take(gdn):
    # checked before any pointer is taken or anything is launched (CPU tensors suffice here)
    import torch
    from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
    x = make_inputs(workload("batched_verify", B=2))
    args = lambda **kw: [kw.get(n, x[n]) for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias")]
    st = x["S0"]
    cases = [
        (dict(a=x["a"].float()), {}, "a and b must have q's dtype"),
        (dict(A_log=x["A_log"].double()), {}, "A_log must be float32"),
        ({}, dict(accept_len=x["accept_len"].long()), "accept_len must be int32"),
        ({}, dict(state_in=st.double()), "state_in must be float32"),
        ({}, dict(o=torch.empty(x["v"].shape, dtype=torch.bfloat16)), "o is torch.bfloat16"),
    ]
    for over, kw, msg in cases:
        call = dict(state_in=st, accept_len=x["accept_len"])
        call.update(kw)
        with pytest.raises(TypeError, match=msg):
            gdn.verify_step(*args(**over), call.pop("state_in"), **call)
    with pytest.raises(TypeError, match="state must be float32"):
        gdn.decode_step(*args(), st.half())
    with pytest.raises(TypeError, match="state_out must be float32"):
        gdn.chunk_prefill(*args(), None, st.double())


def test_binding_rejects_a_tensor_on_another_device(gdn, monkeypatch):
    # Kernels run on the current device's stream: a tensor on another GPU is refused before
    # its pointer is taken. Emulated on the CPU with a stand-in for a cuda:1 tensor while
    # cuda:0 is current.
    import torch

    class OnDevice1:
        is_cuda = True

        def is_contiguous(self):
            return True

        def get_device(self):
            return 1

        def data_ptr(self):
            raise AssertionError("pointer taken before the device check")

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="cuda:1 but the current CUDA device is cuda:0"):
        gdn._ptr(OnDevice1())
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)

    class Ok(OnDevice1):
        def data_ptr(self):
            return 0x1000

    assert gdn._ptr(Ok()) == 0x1000


def test_launch_flags_are_validated_on_the_host(gdn):
    # GDN_LAUNCH_PDL (bit 0) is the only flag; any other bit is rejected before a launch, and
    # the binding passes the flag through the shape.
    INVALID = -1
    assert gdn.GDN_LAUNCH_PDL == 1
    sh = gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128, launch_flags=2)
    assert sh.launch_flags == 2
    assert _call_verify(gdn, sh) == INVALID
    assert "launch_flags" in gdn.lib().gdn_last_error().decode()
    sh = gdn.make_shape(B=2, T=8, H_k=16, H_v=48, d_k=128, d_v=128, launch_flags=gdn.GDN_LAUNCH_PDL | 4)
    assert _call_verify(gdn, sh) == INVALID


def test_selftests_validate_on_the_host(gdn):
    INVALID = -1
    lib = gdn.lib()
    fake = 0x10000
    assert lib.gdn_selftest_accept_wait(None, fake, 16, None) == INVALID
    assert lib.gdn_selftest_accept_wait(fake, None, 16, None) == INVALID
    assert lib.gdn_selftest_accept_wait(fake + 2, fake, 16, None) == INVALID      # misaligned
    assert lib.gdn_selftest_accept_wait(fake, fake, 0, None) == INVALID
    assert lib.gdn_selftest_accept_wait(fake, fake, (1 << 20) + 1, None) == INVALID
    assert "polls" in lib.gdn_last_error().decode()
    assert lib.gdn_selftest_bounded_wait(fake, 0, None) == INVALID
