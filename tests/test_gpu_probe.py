"""The read-only HBM probe (a measurement utility) receives every chunk: the
XOR of its per-CTA folds equals the XOR of the first 16 bytes of every 32 KB
chunk of the buffer."""
import numpy as np
import pytest
import torch

import paged_kv_cache_477_b200 as pkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk", [4096, 32768])
@pytest.mark.parametrize("nbytes,nsink", [(16, 1), (4096 + 48, 3), ((1 << 22) + 32768 + 160, 5), (1 << 22, 296)])
def test_hbm_read_probe_folds_every_chunk(nbytes, nsink, chunk):
    assert torch.cuda.is_available()
    g = torch.Generator().manual_seed(nbytes)
    host = torch.randint(0, 256, (nbytes,), generator=g, dtype=torch.uint8)
    buf = host.cuda()
    sink = torch.zeros(nsink, dtype=torch.int32, device="cuda")
    pkv.hbm_read_probe(buf, sink, chunk)
    assert pkv.last_launch_count() == 1
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32))
    words = host.numpy().view(np.uint32)
    firsts = np.concatenate([words[c // 4:c // 4 + 4] for c in range(0, nbytes, chunk)])
    want = np.bitwise_xor.reduce(firsts)
    assert got == want


def test_hbm_read_probe_rejects_bad_sizes():
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError):
        pkv.hbm_read_probe(torch.zeros(24, dtype=torch.uint8, device="cuda"), sink)
    for chunk in (2048, 5000, 65536):
        with pytest.raises(pkv.PagedKVError):
            pkv.hbm_read_probe(torch.zeros(4096, dtype=torch.uint8, device="cuda"), sink, chunk)
