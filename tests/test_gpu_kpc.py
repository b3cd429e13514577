"""GPU parity of per-channel K grouping (KV-cache page, INT8 item: the Key is
quantized per channel; the oracle's reading R16: blocks of 32 tokens, one
(s, z) per channel and block): K codes and block meta written by
kvq_quantize_append byte for byte equal to the oracle's, V per token as
before."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import f16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
TB = 32


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def _alloc(kvq, B, H, cap, bits, G):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, cap, bits, G, DEV, k_axis=kvq.KVQ_AXIS_CHANNEL)
    c.k_codes.fill_(0xA5)
    c.v_codes.fill_(0x5A)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


@pytest.mark.parametrize("H,T", [(2, 64), (4, 160)])  # V rows per sequence 128 / 640
@pytest.mark.parametrize("bits,G", [(4, 64), (8, 128), (2, 32), (4, 32)])
def test_quantize_channels_bit_exact(kvq, bits, G, H, T):
    B, cap = 4, 192
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    k[0, 0, 3, 5] = 300.0  # an outlier inside one channel's block
    c = _alloc(kvq, B, H, cap, bits, G)
    start = [0, 32, 5, 96]  # sequence 2 is off a block boundary: left untouched
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [min(s + T, cap) if s % TB == 0 else s for s in start]
    kc, km = oracle.quantize_cache_channels(f16_bits(k), bits)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits)
    for b, st in enumerate(start):
        if st % TB:
            assert (c.k_codes[b] == 0xA5).all() and (c.v_codes[b] == 0x5A).all()
            assert (c.k_meta[b].view(torch.int16) == -1).all()
            continue
        n = min(T, cap - st)
        p = slice(st, st + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n])
        blk = slice(st // TB, (st + n) // TB)
        assert np.array_equal(c.k_meta[b, :, blk].cpu().numpy().view(np.uint16),
                              km[b, :, :n // TB])
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n])
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vm[b, :, :n])
        assert (c.k_codes[b, :, :st] == 0xA5).all()
        assert (c.k_meta[b, :, :st // TB].view(torch.int16) == -1).all()
