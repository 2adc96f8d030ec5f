"""Host-side checks of the Python binding on caller-supplied buffers (CPU only).

The kernels write outputs at offsets computed from the problem sizes, so an `out`, `lse`,
`dq`/`dk`/`dv` or workspace of the wrong shape, dtype, device or layout must be refused
before anything is launched. A stand-in for a CUDA tensor (shape, dtype, device, layout,
no memory) lets these checks run without a GPU: it fails the test if the binding ever
takes its data pointer, which only happens after every check has passed."""
import pytest
import torch

import io_aware_exact_28_b200 as fa


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's argument checks."""

    def __init__(self, shape, dtype=torch.float16, index=0, contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True
        self._contiguous = contiguous

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return self._contiguous

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return self.dtype.itemsize

    def data_ptr(self):
        raise AssertionError("a data pointer was taken before the checks refused the call")


H16, F32 = torch.float16, torch.float32


def fwd_args(**over):
    a = dict(q=FakeCuda((2, 4, 96, 64)), k=FakeCuda((2, 2, 80, 64)), v=FakeCuda((2, 2, 80, 64)),
             out=FakeCuda((2, 4, 96, 64)), lse=FakeCuda((2, 4, 96), F32))
    a.update(over)
    return a


@pytest.mark.parametrize("bad, err", [
    (dict(out=FakeCuda((2, 4, 96, 32))), ValueError),                 # wrong shape
    (dict(out=FakeCuda((2, 4, 96, 64), torch.bfloat16)), TypeError),  # wrong dtype
    (dict(out=FakeCuda((2, 4, 96, 64), index=1)), ValueError),        # other device
    (dict(out=FakeCuda((2, 4, 96, 64), contiguous=False)), ValueError),
    (dict(lse=FakeCuda((2, 4, 95), F32)), ValueError),
    (dict(lse=FakeCuda((2, 4, 96), H16)), TypeError),
])
def test_fwd_refuses_bad_outputs(bad, err):
    a = fwd_args(**bad)
    with pytest.raises(err):
        fa.fwd(a["q"], a["k"], a["v"], causal=True, out=a["out"], lse=a["lse"])
    with pytest.raises(err):
        fa.fwd_kvcache(a["q"], a["k"], a["v"], 80, out=a["out"], lse=a["lse"])


def test_fwd_paged_refuses_bad_outputs():
    q = FakeCuda((2, 4, 96, 64))
    pool = FakeCuda((40, 2, 16, 64))
    table = FakeCuda((2, 8), torch.int32)
    with pytest.raises(ValueError):
        fa.fwd_paged(q, pool, pool, table, 100, out=FakeCuda((2, 4, 97, 64)),
                     lse=FakeCuda((2, 4, 96), F32))
    with pytest.raises(TypeError):
        fa.fwd_paged(q, pool, pool, table, 100, out=FakeCuda((2, 4, 96, 64)),
                     lse=FakeCuda((2, 4, 96), torch.float64))


def test_fwd_fp8_refuses_bad_outputs():
    q8 = FakeCuda((1, 4, 64, 128), torch.uint8)
    k8 = FakeCuda((1, 2, 64, 128), torch.uint8)
    with pytest.raises(TypeError):       # the FP8 path writes bf16
        fa.fwd_fp8(q8, k8, k8, 1.0, 1.0, 1.0, out=FakeCuda((1, 4, 64, 128), H16),
                   lse=FakeCuda((1, 4, 64), F32))
    with pytest.raises(ValueError):
        fa.fwd_fp8(q8, k8, k8, 1.0, 1.0, 1.0, out=FakeCuda((1, 4, 64, 128), torch.bfloat16),
                   lse=FakeCuda((1, 4, 63), F32))


def bwd_call(**over):
    a = dict(q=FakeCuda((1, 4, 64, 64)), k=FakeCuda((1, 2, 64, 64)), v=FakeCuda((1, 2, 64, 64)),
             o=FakeCuda((1, 4, 64, 64)), lse=FakeCuda((1, 4, 64), F32),
             dout=FakeCuda((1, 4, 64, 64)), dq=FakeCuda((1, 4, 64, 64)),
             dk=FakeCuda((1, 2, 64, 64)), dv=FakeCuda((1, 2, 64, 64)),
             workspace=FakeCuda((1 << 20,), torch.uint8))
    a.update(over)
    return fa.bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], causal=True, dq=a["dq"],
                  dk=a["dk"], dv=a["dv"], workspace=a["workspace"])


@pytest.mark.parametrize("bad, err", [
    (dict(lse=FakeCuda((1, 4, 32), F32)), ValueError),
    (dict(lse=FakeCuda((1, 4, 64), H16)), TypeError),
    (dict(dq=FakeCuda((1, 2, 64, 64))), ValueError),       # dq takes q's shape
    (dict(dk=FakeCuda((1, 4, 64, 64))), ValueError),       # dk takes k's shape
    (dict(dv=FakeCuda((1, 2, 64, 64), torch.bfloat16)), TypeError),
    (dict(workspace=FakeCuda((1 << 20,), torch.uint8, index=1)), ValueError),
    (dict(workspace=FakeCuda((1 << 20,), torch.uint8, contiguous=False)), ValueError),
])
def test_bwd_refuses_bad_buffers(bad, err):
    with pytest.raises(err):
        bwd_call(**bad)


def decode_args(**over):
    a = dict(q=FakeCuda((3, 8, 128)), kc=FakeCuda((3, 2, 512, 128)), vc=FakeCuda((3, 2, 512, 128)),
             lens=FakeCuda((3,), torch.int32), out=FakeCuda((3, 8, 128)),
             lse=FakeCuda((3, 8), F32), workspace=FakeCuda((1 << 22,), torch.uint8))
    a.update(over)
    return a


@pytest.mark.parametrize("bad, err", [
    (dict(out=FakeCuda((3, 8, 64))), ValueError),
    (dict(out=FakeCuda((3, 8, 128), torch.bfloat16)), TypeError),
    (dict(lse=FakeCuda((3, 4), F32)), ValueError),
    (dict(lse=FakeCuda((3, 8), H16)), TypeError),
    (dict(workspace=FakeCuda((1 << 22,), torch.uint8, index=2)), ValueError),
])
def test_decode_refuses_bad_buffers(bad, err):
    a = decode_args(**bad)
    with pytest.raises(err):
        fa.decode(a["q"], a["kc"], a["vc"], a["lens"], out=a["out"], lse=a["lse"],
                  workspace=a["workspace"])
    if "workspace" not in bad:
        with pytest.raises(err):
            fa.decode_noalloc(a["q"], a["kc"], a["vc"], a["lens"], out=a["out"], lse=a["lse"])


def test_decode_paged_refuses_bad_buffers():
    q = FakeCuda((3, 8, 128))
    pool = FakeCuda((64, 2, 16, 128))
    table = FakeCuda((3, 32), torch.int32)
    lens = FakeCuda((3,), torch.int32)
    good = dict(out=FakeCuda((3, 8, 128)), lse=FakeCuda((3, 8), F32),
                workspace=FakeCuda((1 << 22,), torch.uint8))
    for bad, err in ((dict(out=FakeCuda((3, 8, 127))), ValueError),
                     (dict(lse=FakeCuda((3, 8), torch.float64)), TypeError),
                     (dict(workspace=FakeCuda((1 << 22,), torch.uint8, contiguous=False)), ValueError)):
        a = dict(good, **bad)
        with pytest.raises(err):
            fa.decode_paged(q, pool, pool, table, lens, out=a["out"], lse=a["lse"],
                            workspace=a["workspace"])


def test_launch_makes_the_tensors_device_current_and_passes_its_stream(monkeypatch):
    """`_launch` enters the tensors' device, takes that device's current stream unless one
    is given, and appends its handle as the last argument of the entry point."""
    events = []

    class Dev:
        def __init__(self, device):
            self.device = device

        def __enter__(self):
            events.append(("enter", self.device))

        def __exit__(self, *exc):
            events.append(("exit", self.device))
            return False

    class Stream:
        def __init__(self, handle, device=torch.device("cuda", 1)):
            self.cuda_stream = handle
            self.device = device

    monkeypatch.setattr(torch.cuda, "device", Dev)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: Stream(4242))
    calls = []

    def entry(*args):
        calls.append(args)
        events.append(("call", None))
        return 0

    dev1 = torch.device("cuda", 1)
    assert fa._launch(dev1, None, entry, 11, 22) == 0
    assert calls[-1] == (11, 22, 4242)
    assert events == [("enter", dev1), ("call", None), ("exit", dev1)]
    assert fa._launch(dev1, Stream(7), entry, 5) == 0
    assert calls[-1] == (5, 7)


def test_launch_records_owned_tensors_on_a_side_stream(monkeypatch):
    """Tensors the wrapper allocated come from the current stream's pool; when the kernels
    run on another stream they are recorded on it (so the allocator does not reuse their
    memory while those kernels may still run), and a stream of another device is refused
    before anything is launched."""
    class Dev:
        def __init__(self, device):
            pass

        def __enter__(self):
            return None

        def __exit__(self, *exc):
            return False

    class Stream:
        def __init__(self, handle, device):
            self.cuda_stream = handle
            self.device = device

    class Owned:
        def __init__(self):
            self.recorded = []

        def record_stream(self, s):
            self.recorded.append(s.cuda_stream)

    dev0 = torch.device("cuda", 0)
    monkeypatch.setattr(torch.cuda, "device", Dev)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: Stream(100, dev0))
    calls = []

    def entry(*args):
        calls.append(args)
        return 0

    a, b = Owned(), Owned()
    fa._launch(dev0, None, entry, 1, owned=[a, None, b])        # current stream: nothing to record
    assert a.recorded == [] and b.recorded == []
    fa._launch(dev0, Stream(100, dev0), entry, 1, owned=[a])     # the current stream, passed in
    assert a.recorded == []
    fa._launch(dev0, Stream(555, dev0), entry, 2, owned=[a, None, b])
    assert calls[-1] == (2, 555) and a.recorded == [555] and b.recorded == [555]
    n = len(calls)
    with pytest.raises(ValueError):
        fa._launch(dev0, Stream(9, torch.device("cuda", 3)), entry, 3, owned=[a])
    assert len(calls) == n and a.recorded == [555]


def test_wrappers_hand_their_own_allocations_to_launch(monkeypatch):
    """Each wrapper lists exactly the tensors it allocated (outputs it was not given, the
    workspace) as owned; caller-supplied buffers are not listed."""
    seen = {}

    def capture(device, stream, fn, *args, owned=()):
        seen[fn.__name__] = list(owned)
        return fa.FA_OK

    made = []

    def fake_empty(*shape, dtype=None, device=None, **kw):
        t = ValidFake(shape[0] if len(shape) == 1 and isinstance(shape[0], (tuple, list, torch.Size)) else shape,
                      dtype or torch.float32)
        made.append(t)
        return t

    def fake_empty_like(x, **kw):
        t = ValidFake(tuple(x.shape), x.dtype)
        made.append(t)
        return t

    monkeypatch.setattr(fa, "_launch", capture)
    monkeypatch.setattr(torch, "empty", fake_empty)
    monkeypatch.setattr(torch, "empty_like", fake_empty_like)
    monkeypatch.setattr(fa, "decode_workspace_bytes", lambda *a: 1 << 20)
    monkeypatch.setattr(fa, "bwd_workspace_bytes", lambda *a: 1 << 20)
    V = ValidFake
    q4, k4 = V((2, 4, 96, 64)), V((2, 2, 80, 64))
    o, l = fa.fwd(q4, k4, k4)
    assert seen["fa_fwd"] == [o, l]
    given = V((2, 4, 96, 64))
    o, l = fa.fwd(q4, k4, k4, out=given)
    assert o is given and seen["fa_fwd"] == [l]
    q3, cache, lens = V((3, 8, 128)), V((3, 2, 512, 128)), V((3,), torch.int32)
    made.clear()
    fa.decode(q3, cache, cache, lens)
    assert seen["fa_decode"] == made and len(made) == 3     # out, lse, workspace
    made.clear()
    fa.decode(q3, cache, cache, lens, workspace=V((1 << 22,), torch.uint8), return_lse=False)
    assert seen["fa_decode"] == made and len(made) == 1     # out only
    qb, kb = V((1, 4, 64, 64)), V((1, 2, 64, 64))
    made.clear()
    fa.bwd(qb, kb, kb, V((1, 4, 64, 64)), V((1, 4, 64), F32), V((1, 4, 64, 64)))
    assert seen["fa_bwd"] == made and len(made) == 4        # dq, dk, dv, workspace


class ValidFake(FakeCuda):
    """A stand-in that passes every check and hands out a distinct fake address."""
    _next = 0x10000

    def data_ptr(self):
        ValidFake._next += 0x1000
        return ValidFake._next


def test_every_entry_point_receives_its_declared_argument_count(monkeypatch):
    """Each binding function passes exactly the arguments its C entry point declares (the
    stream handle is appended last by `_launch`)."""
    seen = {}

    def capture(device, stream, fn, *args, owned=()):
        seen[fn.__name__] = (len(args) + 1, len(fn.argtypes), args)
        return fa.FA_OK

    monkeypatch.setattr(fa, "_launch", capture)
    V = ValidFake
    q4, k4 = V((2, 4, 96, 64)), V((2, 2, 80, 64))
    fa.fwd(q4, k4, k4, out=V((2, 4, 96, 64)), lse=V((2, 4, 96), F32))
    fa.fwd_kvcache(q4, k4, k4, 80, out=V((2, 4, 96, 64)), lse=V((2, 4, 96), F32))
    pool, table = V((40, 2, 16, 64)), V((2, 8), torch.int32)
    fa.fwd_paged(q4, pool, pool, table, 100, out=V((2, 4, 96, 64)), lse=V((2, 4, 96), F32))
    q8, k8 = V((1, 4, 64, 128), torch.uint8), V((1, 2, 64, 128), torch.uint8)
    fa.fwd_fp8(q8, k8, k8, 1.0, 1.0, 1.0, out=V((1, 4, 64, 128), torch.bfloat16),
               lse=V((1, 4, 64), F32))
    qb, kb = V((1, 4, 64, 64)), V((1, 2, 64, 64))
    fa.bwd(qb, kb, kb, V((1, 4, 64, 64)), V((1, 4, 64), F32), V((1, 4, 64, 64)),
           dq=V((1, 4, 64, 64)), dk=V((1, 2, 64, 64)), dv=V((1, 2, 64, 64)),
           workspace=V((1 << 20,), torch.uint8))
    q3, cache, lens = V((3, 8, 128)), V((3, 2, 512, 128)), V((3,), torch.int32)
    fa.decode(q3, cache, cache, lens, out=V((3, 8, 128)), lse=V((3, 8), F32),
              workspace=V((1 << 22,), torch.uint8))
    fa.decode_noalloc(q3, cache, cache, lens, out=V((3, 8, 128)), lse=V((3, 8), F32))
    dpool, dtable = V((64, 2, 16, 128)), V((3, 32), torch.int32)
    fa.decode_paged(q3, dpool, dpool, dtable, lens, out=V((3, 8, 128)), lse=V((3, 8), F32),
                    workspace=V((1 << 22,), torch.uint8))
    assert set(seen) == {"fa_fwd", "fa_fwd_kvcache", "fa_fwd_paged", "fa_fwd_fp8", "fa_bwd",
                         "fa_decode", "fa_decode_noalloc", "fa_decode_paged"}
    for name, (passed, declared, _) in seen.items():
        assert passed == declared, (name, passed, declared)
    # spot checks of sizes in their places
    assert seen["fa_fwd"][2][5:11] == (2, 4, 2, 96, 80, 64)
    assert seen["fa_decode"][2][6:11] == (3, 8, 2, 512, 128)
    assert seen["fa_decode_paged"][2][7:13] == (3, 8, 2, 64, 16, 32)
    assert seen["fa_fwd_kvcache"][2][3:5] == (None, None)
    assert seen["fa_fwd_kvcache"][2][7:13] == (2, 4, 2, 96, 80, 80)
    assert seen["fa_fwd_paged"][2][4:6] == (None, None)
    assert seen["fa_fwd_paged"][2][8:16] == (2, 4, 2, 96, 100, 40, 16, 8)
    # per-sequence lengths ride in their own slots
    ql, kl = V((2,), torch.int32), V((2,), torch.int32)
    fa.fwd_kvcache(q4, k4, k4, 80, out=V((2, 4, 96, 64)), lse=V((2, 4, 96), F32), q_lens=ql,
                   kv_lens=kl)
    assert all(isinstance(x, int) for x in seen["fa_fwd_kvcache"][2][3:5])
    assert seen["fa_fwd_kvcache"][0] == seen["fa_fwd_kvcache"][1]


def test_per_sequence_lengths_are_checked():
    q4, k4 = FakeCuda((2, 4, 96, 64)), FakeCuda((2, 2, 80, 64))
    for bad, err in ((FakeCuda((3,), torch.int32), TypeError),          # one per sequence
                     (FakeCuda((2,), torch.int64), TypeError),          # int32 only
                     (FakeCuda((2,), torch.int32, index=1), ValueError)):
        with pytest.raises(err):
            fa.fwd_kvcache(q4, k4, k4, 80, q_lens=bad, out=FakeCuda((2, 4, 96, 64)),
                           lse=FakeCuda((2, 4, 96), F32))
        with pytest.raises(err):
            fa.fwd_paged(q4, FakeCuda((40, 2, 16, 64)), FakeCuda((40, 2, 16, 64)),
                         FakeCuda((2, 8), torch.int32), 100, kv_lens=bad,
                         out=FakeCuda((2, 4, 96, 64)), lse=FakeCuda((2, 4, 96), F32))
