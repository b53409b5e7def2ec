"""The binding's checks of tensor arguments, on the CPU.

The C entry points take bare device addresses; the binding refuses, before
any library call, a tensor the kernels could not safely use: host memory, a
non-contiguous view, another device than the cache's, or fewer bytes than
the call reads or writes.  A stand-in object plays the CUDA tensor here (no
GPU in this suite).  A call that passes the checks reaches the library with
a null cache handle, which the library refuses on the host."""
import pytest
import torch

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import SINGLE_480P

W = SINGLE_480P.scaled(layers=1, kv_heads=4, action_tokens=4)
# bytes per rollout: q/out F*T*H*d*2, block k/v F*Tf*Hkv*d*2, lse H*F*T*4
Q_BYTES = 3 * 1560 * 12 * 128 * 2
KV_BYTES = 3 * 1564 * 4 * 128 * 2
LSE_BYTES = 12 * 3 * 1560 * 4


class FakeCuda:
    """Duck-typed CUDA tensor: bytes, contiguity and device, no memory."""

    def __init__(self, nbytes, contiguous=True, device="cuda:0", esz=2):
        self.nbytes, self.contiguous, self.esz = nbytes, contiguous, esz
        self.device = torch.device(device)
        self.is_cuda = self.device.type == "cuda"

    def is_contiguous(self):
        return self.contiguous

    def numel(self):
        return self.nbytes // self.esz

    def element_size(self):
        return self.esz

    def data_ptr(self):
        return 256


def _cache():
    c = fd.Cache.__new__(fd.Cache)
    c.desc = fd.make_desc(W)
    c.storage = FakeCuda(1 << 20, esz=1)
    c.handle = None
    return c


def _attn_args(n=2, **over):
    a = dict(q=FakeCuda(n * Q_BYTES), k=FakeCuda(n * KV_BYTES), v=FakeCuda(n * KV_BYTES),
             out=FakeCuda(n * Q_BYTES), lse=FakeCuda(n * LSE_BYTES, esz=4))
    a.update(over)
    return a


@pytest.mark.parametrize("entry", [fd.fd_block_attention, fd.fd_block_attention_static])
@pytest.mark.parametrize("name,bad,status", [
    ("q", torch.zeros(4), 1),                                   # host tensor
    ("k", FakeCuda(2 * KV_BYTES, contiguous=False), 1),         # strided view
    ("v", FakeCuda(2 * KV_BYTES, device="cuda:1"), 1),          # another GPU
    ("out", FakeCuda(2 * Q_BYTES - 2), 2),                      # one element short
    ("lse", FakeCuda(2 * LSE_BYTES - 4, esz=4), 2),
    ("k", FakeCuda(1 * KV_BYTES), 2),                           # sized for one rollout
])
def test_attention_refuses_unusable_tensors(entry, name, bad, status):
    with pytest.raises(fd.FdError) as e:
        entry(_cache(), 0, 2, **_attn_args(**{name: bad}))
    assert e.value.status == status
    assert name in str(e.value)


def test_attention_sizes_accept_exact_buffers():
    """Exactly sized tensors pass every check and reach the library (which
    refuses the null cache handle: FD_ERR_INVALID_ARG from the C side)."""
    with pytest.raises(fd.FdError) as e:
        fd.fd_block_attention(_cache(), 0, 2, **_attn_args(), stream=0)
    assert str(e.value) == "fd_block_attention: FD_ERR_INVALID_ARG"


def test_commit_checks_lists_and_sizes():
    c = _cache()
    ok = [FakeCuda(2 * KV_BYTES)]
    with pytest.raises(fd.FdError, match="for 1 layers"):
        fd.fd_cache_commit(c, 0, 1, 2, ok + ok, ok)
    with pytest.raises(fd.FdError, match="frame counts"):
        fd.fd_cache_commit(c, 0, 1, 2, ok, ok, frames=[1])
    with pytest.raises(fd.FdError, match=r"v\[0\] holds"):
        fd.fd_cache_commit(c, 0, 1, 2, ok, [FakeCuda(2 * KV_BYTES - 16)])
    with pytest.raises(fd.FdError, match="not a CUDA tensor"):
        fd.fd_cache_commit(c, 0, 1, 2, [torch.zeros(8)], ok)


def test_rope3d_checks_size_of_its_tensor():
    # x [R][F][Tx][heads][d]: 2 rollouts of the block keys (Tx = Tf, Hkv heads)
    with pytest.raises(fd.FdError) as e:
        fd.fd_rope3d(_cache(), 0, 2, FakeCuda(2 * KV_BYTES - 2), 1564, 4)
    assert e.value.status == 2


def test_combine_checks_parts():
    out = torch.zeros((1, 8, 2, 16))            # host tensor
    with pytest.raises(fd.FdError, match="2 row tensors, 1 lse"):
        fd.fd_attention_combine([out, out], [out], out)
    with pytest.raises(fd.FdError, match="not a CUDA tensor"):
        fd.fd_attention_combine([out], [torch.zeros((1, 2, 8))], out)
