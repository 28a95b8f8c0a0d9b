"""GPU tests of decode-on-use (ECF8 walkthrough §3.2.2: a fixed pool reused
cyclically, each layer decoded when its forward pass needs it; DFloat11
article §4: decode ahead in the background while the current layer
computes).  The result is defined by the codec being lossless: whatever the
schedule, the weights a layer's consumer reads are exactly its source bytes,
and an FP8 GEMM over them equals the GEMM over the source weights."""
import numpy as np
import pytest

import ecf8_synth as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    import lossless_fp8_weight_b200 as L
    return L, torch


# a 1-bit-code (wide table) tensor kind and two others, so every layer mixes
# both table widths in one launch
SPECS = [synth.alpha_sweep_point(1.7, 448.0).tensors[0], synth.alpha_sweep_point(1.5, 448.0).tensors[0],
         synth.alpha_sweep_point(2.0, 28.0).tensors[0]]


def _layers(L, torch, n_layers, seed, sizes=None):
    r = np.random.default_rng(seed)
    layers, srcs = [], []
    for _ in range(n_layers):
        tensors, xs, off = [], [], 0
        for k, spec in enumerate(SPECS):
            n = int(r.integers(20_000, 300_000)) if sizes is None else sizes[k]
            x = spec.generate(begin=int(r.integers(0, 1 << 24)), count=n)
            blob = L.encode(x)
            tensors.append(L.PipelineTensor(L.blob_info(blob), torch.from_numpy(blob).cuda(), off))
            xs.append((off, x))
            off = (off + n + 31) // 32 * 32
        layers.append(tensors)
        srcs.append(xs)
    slot_bytes = max(o + x.size for xs in srcs for o, x in xs)
    return layers, srcs, slot_bytes


def _run_passes(env, n_layers, n_slots, depth, max_ctas, passes=2, seed=11):
    L, torch = env
    layers, srcs, slot_bytes = _layers(L, torch, n_layers, seed)
    slots = [torch.full((slot_bytes,), 0xEE, dtype=torch.uint8, device="cuda") for _ in range(n_slots)]
    by_ptr = {s.data_ptr(): s for s in slots}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    compute, decode = torch.cuda.Stream(), torch.cuda.Stream()
    P = L.Pipeline(layers, slots, slot_bytes, depth=depth, max_ctas=max_ctas, status=status, decode_stream=decode)
    got = []
    for _ in range(passes):
        for l in range(n_layers):
            slot = by_ptr[P.acquire(l, compute)]
            with torch.cuda.stream(compute):
                got.append((l, [slot[o:o + x.size].clone() for o, x in srcs[l]]))
            P.release(l, compute)
    torch.cuda.synchronize()
    P.close()
    assert int(status.item()) == 0
    for l, outs in got:
        for (o, x), d in zip(srcs[l], outs):
            assert np.array_equal(d.cpu().numpy(), x), (l, o)


@pytest.mark.parametrize("n_slots,depth,max_ctas", [(2, 1, 0), (3, 2, 0), (2, 1, 7), (1, 0, 0), (4, 1, 32)])
def test_every_layer_reads_its_source_bytes(env, n_slots, depth, max_ctas):
    _run_passes(env, n_layers=7, n_slots=n_slots, depth=depth, max_ctas=max_ctas)


def test_fp8_gemm_over_decoded_weights_equals_gemm_over_source(env):
    """The consumer the pages pair with the decode: y = x W^T in FP8, on the
    compute stream, with W read from the pipeline's slot."""
    L, torch = env
    if not hasattr(torch, "_scaled_mm"):
        pytest.skip("torch._scaled_mm missing")
    N, K, M = 256, 512, 128
    layers, srcs, slot_bytes = _layers(L, torch, 4, seed=5, sizes=[N * K, N * K, N * K])
    slots = [torch.empty(slot_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    by_ptr = {s.data_ptr(): s for s in slots}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    compute, decode = torch.cuda.Stream(), torch.cuda.Stream()
    P = L.Pipeline(layers, slots, slot_bytes, depth=1, status=status, decode_stream=decode)
    x = torch.from_numpy(SPECS[0].generate(begin=7, count=M * K)).cuda().view(torch.float8_e4m3fn).view(M, K)
    one = torch.ones((), dtype=torch.float32, device="cuda")
    ys = []
    for l in range(4):
        slot = by_ptr[P.acquire(l, compute)]
        with torch.cuda.stream(compute):
            for o, _ in srcs[l]:
                w = slot[o:o + N * K].view(torch.float8_e4m3fn).view(N, K)
                ys.append(torch._scaled_mm(x, w.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
        P.release(l, compute)
    torch.cuda.synchronize()
    P.close()
    assert int(status.item()) == 0
    k = 0
    for l in range(4):
        for _, src in srcs[l]:
            w = torch.from_numpy(src).cuda().view(torch.float8_e4m3fn).view(N, K)
            want = torch._scaled_mm(x, w.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            assert torch.equal(ys[k], want), (l, k)
            k += 1


def test_capped_grid_decodes_the_same_bytes(env):
    L, torch = env
    xs = [s.generate(begin=3, count=500_000 + 17 * i) for i, s in enumerate(SPECS)]
    blobs = [L.encode(x) for x in xs]
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).cuda() for b in blobs]
    for cap in (1, 2, 5, 148, 10_000):
        outs = [torch.empty(i.n, dtype=torch.uint8, device="cuda") for i in infos]
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.decode_batched([L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, outs)], status=status,
                         max_ctas=cap)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for x, o in zip(xs, outs):
            assert np.array_equal(o.cpu().numpy(), x), cap


def test_acquiring_into_a_slot_still_in_use_is_refused(env):
    L, torch = env
    layers, srcs, slot_bytes = _layers(L, torch, 3, seed=9)
    slots = [torch.empty(slot_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    compute, decode = torch.cuda.Stream(), torch.cuda.Stream()
    P = L.Pipeline(layers, slots, slot_bytes, depth=1, status=status, decode_stream=decode)
    P.acquire(0, compute)
    with pytest.raises(L.Ecf8Error) as e:
        P.acquire(2, compute)  # slot 0 still holds layer 0
    assert e.value.code == -1
    with pytest.raises(L.Ecf8Error):
        P.release(1, compute)  # layer 1 was decoded ahead but never acquired
    P.release(0, compute)
    P.acquire(1, compute)
    P.release(1, compute)
    P.acquire(2, compute)
    P.release(2, compute)
    torch.cuda.synchronize()
    P.close()
    assert int(status.item()) == 0
