"""CPU checks of the Python binding's tensor validation.  The C ABI sees raw
pointers only, so the binding must reject host tensors, tensors of another
device, non-contiguous views and wrong dtypes or shapes before any call.  Valid
argument sets are checked with stand-in CUDA tensor objects and a recording
stand-in for the library, so that no check rejects what the GPU tests, the
smoke check and the bench pass."""
import types

import pytest

torch = pytest.importorskip("torch")
import mask_aware_flash_b200 as fm  # noqa: E402


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's checks and marshalling."""

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True, ptr=0x10000):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = True
        self._contiguous = contiguous
        self._ptr = ptr

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def data_ptr(self):
        return self._ptr

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        return 1 if self.dtype == torch.uint8 else 4


class Recorder:
    """Stands in for the loaded library: every entry point returns FM_OK and is recorded."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            if name == "fm_status_string":  # used by FmError's message, not a compute call
                return b"stand-in status"
            self.calls.append(name)
            return 1024 if name.endswith("_bytes") else fm.FM_OK
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(fm, "lib", lambda: r)
    return r


STREAM = types.SimpleNamespace(cuda_stream=0)
B, NQ, NK, H, HKV, D = 2, 300, 512, 4, 2, 128


def _meta(Hm=1):
    m = fm.MaskMeta.__new__(fm.MaskMeta)
    m.desc = fm.MaskDesc(B, Hm, NQ, NK, 128, 128)
    m.c = fm.MaskMetaC()
    return m


def _qkv(dtype=torch.bfloat16):
    return (FakeCuda((B, NQ, H, D), dtype), FakeCuda((B, NK, HKV, D), dtype), FakeCuda((B, NK, HKV, D), dtype))


def _vecs(Hm=1, n=NK):
    return [FakeCuda((B, Hm, n), torch.int32) for _ in range(3)] + [None]


def test_valid_forward_and_backward_reach_the_library(rec):
    q, k, v = _qkv()
    o, lse = FakeCuda(q.shape, q.dtype), FakeCuda((B, H, NQ), torch.float32)
    fm.fm_attn_fwd(q, k, v, _meta(), _vecs(), 0.1, o=o, lse=lse, stream=STREAM)
    do, dq = FakeCuda(q.shape, q.dtype), FakeCuda(q.shape, q.dtype)
    dk, dv = FakeCuda(k.shape, k.dtype), FakeCuda(k.shape, k.dtype)
    ws = FakeCuda((1024,), torch.uint8)
    fm.fm_attn_bwd(q, k, v, o, lse, do, _meta(H), _vecs(H), 0.1, dq=dq, dk=dk, dv=dv, ws=ws, stream=STREAM,
                   deterministic=True)
    q32, k32, v32 = (FakeCuda(t.shape[:3] + (64,), torch.float32) for t in _qkv())
    fm.fm_attn_fwd(q32, k32, v32, _meta(), _vecs(), 0.1, o=FakeCuda(q32.shape, torch.float32), lse=lse,
                   stream=STREAM)
    assert rec.calls == ["fm_attn_fwd", "fm_attn_bwd_workspace_bytes", "fm_attn_bwd", "fm_attn_fwd"]


def test_valid_integer_passes_reach_the_library(rec):
    v = [FakeCuda((B, 1, NK), torch.int32) for _ in range(4)]
    out = [FakeCuda((3, B, 1, NK), torch.int32) for _ in range(4)]
    fm.fm_localize(v, [[0], [128], [256]], [[128]] * 3, out=out, stream=STREAM)
    fm.fm_kv_chunk_pairs(out, [128] * 3, 100, out=FakeCuda((3, B, 1, 6), torch.int64), stream=STREAM)
    fm.fm_varlen_mask(FakeCuda((5,), torch.int32), 700, out=[FakeCuda((1, 1, 700), torch.int32) for _ in range(4)],
                      stream=STREAM)
    assert rec.calls == ["fm_localize", "fm_kv_chunk_pairs", "fm_varlen_mask"]


@pytest.mark.parametrize("bad", ["host", "device", "view", "dtype", "shape"])
def test_forward_rejects_bad_tensors(rec, bad):
    q, k, v = _qkv()
    o, lse = FakeCuda(q.shape, q.dtype), FakeCuda((B, H, NQ), torch.float32)
    if bad == "host":
        k.is_cuda = False
    elif bad == "device":
        v.device = torch.device("cuda:1")
    elif bad == "view":
        o._contiguous = False
    elif bad == "dtype":
        lse.dtype = torch.float16
    else:
        v.shape = torch.Size((B, NK + 4, HKV, D))
    with pytest.raises(fm.FmError):
        fm.fm_attn_fwd(q, k, v, _meta(), _vecs(), 0.1, o=o, lse=lse, stream=STREAM)
    assert rec.calls == []


def test_backward_rejects_mismatched_gradient_and_vectors(rec):
    q, k, v = _qkv()
    o, lse, do = FakeCuda(q.shape, q.dtype), FakeCuda((B, H, NQ), torch.float32), FakeCuda(q.shape, q.dtype)
    ws = FakeCuda((1024,), torch.uint8)
    with pytest.raises(fm.FmError):  # dk shaped like q
        fm.fm_attn_bwd(q, k, v, o, lse, do, _meta(), _vecs(), 0.1, dq=FakeCuda(q.shape, q.dtype),
                       dk=FakeCuda(q.shape, q.dtype), dv=FakeCuda(k.shape, k.dtype), ws=ws, stream=STREAM)
    with pytest.raises(fm.FmError):  # vectors of another key length than the metadata
        fm.fm_attn_bwd(q, k, v, o, lse, do, _meta(), _vecs(n=NK - 4), 0.1, dq=FakeCuda(q.shape, q.dtype),
                       dk=FakeCuda(k.shape, k.dtype), dv=FakeCuda(k.shape, k.dtype), ws=ws, stream=STREAM)
    assert "fm_attn_bwd" not in rec.calls


def test_real_host_tensors_are_rejected(rec):
    q = torch.zeros((1, 128, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(fm.FmError):
        fm.fm_attn_fwd(q, q, q, _meta(), [None] * 4, 0.1, o=q, lse=torch.zeros((1, 2, 128)), stream=STREAM)
    with pytest.raises(fm.FmError):
        fm.fm_build_mask_meta(torch.zeros((1, 1, 128), dtype=torch.int32), None, None, None, n_q=128)
    with pytest.raises(fm.FmError):
        fm.fm_kv_chunk_pairs([FakeCuda((1, 1, 1, 128), torch.int32)] * 4, [128], 0)  # chunk_len 0
    assert rec.calls == []
