"""GPU encoder parity: the blob ecf8_encode_device writes is byte for byte
the CPU oracle's encoding of the same tensor (ECF8 walkthrough §3.1.1-§3.2.1:
histogram, Huffman code, canonical table, MSB-first code stream with per-chunk
gaps and per-group offsets, raw nibbles), and the GPU histogram is the
exponent count.  Inputs span the edge sizes around the 16-weight thread, the
4096-weight segment and the 32-chunk group, every code-length regime (1-bit
codes, 2+ bits, a single symbol), and two layouts."""
import numpy as np
import pytest

import ecf8_synth as synth
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    import lossless_fp8_weight_b200 as L
    return L, torch


SIZES = [1, 2, 7, 15, 16, 17, 31, 33, 255, 4095, 4096, 4097, 8191, 65537, 300_007]


def _check(env, x, chunk_bytes=32, group_chunks=32):
    L, torch = env
    d = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    h = L.histogram_device(d)
    assert np.array_equal(h, np.bincount((x >> 3) & 15, minlength=16).astype(np.uint64))
    blob = L.encode_device(d, chunk_bytes=chunk_bytes, group_chunks=group_chunks).cpu().numpy()
    want = oracle.encode(x, chunk_bytes=chunk_bytes, group_chunks=group_chunks)
    assert blob.size == want.size
    if not np.array_equal(blob, want):
        i = int(np.flatnonzero(blob != want)[0])
        raise AssertionError(f"first differing byte {i} of {blob.size}: {blob[i]} != {want[i]}")


@pytest.mark.parametrize("n", SIZES)
def test_gaussian_sizes(env, n):
    _check(env, synth.single_normal_1k().tensors[0].generate(count=n))


@pytest.mark.parametrize("alpha,max_abs", [(1.5, 448.0), (1.7, 448.0), (1.7, 112.0), (2.0, 28.0)])
def test_sweep_distributions(env, alpha, max_abs):
    _check(env, synth.alpha_sweep_point(alpha, max_abs).tensors[0].generate(begin=12345, count=1_000_003))


def test_small_layout(env):
    x = synth.alpha_sweep_point(1.9, 448.0).tensors[0].generate(count=70_001)
    _check(env, x, chunk_bytes=4, group_chunks=1)
    _check(env, x, chunk_bytes=8, group_chunks=5)


def test_every_byte_value_and_a_single_symbol(env):
    r = np.random.default_rng(7)
    _check(env, r.permutation(np.repeat(np.arange(256, dtype=np.uint8), 211)))
    _check(env, np.full(50_001, 0x38, dtype=np.uint8))


def test_full_size_ffn_tensor_decodes_after_gpu_encode(env):
    """14336x4096 encoded on the GPU, then decoded by the GPU decoder."""
    L, torch = env
    x = synth.alpha_sweep_point(1.7, 448.0).tensors[0].generate()
    d = torch.from_numpy(x).cuda()
    blob = L.encode_device(d)
    info = L.blob_info(blob.cpu().numpy())
    out = torch.empty(info.n, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.decode(info, blob, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, d)
    assert np.array_equal(blob.cpu().numpy(), L.encode(x))
