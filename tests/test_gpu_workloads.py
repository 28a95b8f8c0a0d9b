"""GPU parity at the workloads' full sizes.

Every decoded byte is compared with the seeded source tensor it came from
(decode(encode(x)) == x is the definition of the result: ECF8 walkthrough §1,
arXiv 2510.02676 abstract), and sampled tensors are also compared with the
CPU oracle's own decode of the same blob.  Blobs come from the library's
encoder, whose bytes equal the oracle's (tests/test_library_host.py).
"""
import concurrent.futures as cf
import hashlib
import os

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


def _encode(L, specs):
    xs, blobs = [], []
    for t in specs:
        x = t.generate()
        xs.append(x)
        blobs.append(L.encode(x))
    return xs, blobs


def _decode_batched(env, blobs, reuse_out=None):
    """One batched launch (workspace path when the batch is large)."""
    L, torch = env
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).cuda() for b in blobs]
    outs = reuse_out if reuse_out is not None else [torch.empty(i.n, dtype=torch.uint8, device="cuda") for i in infos]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(L.batched_workspace_size(len(blobs)), 16), dtype=torch.uint8, device="cuda")
    L.decode_batched([L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, outs)], workspace=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return outs


def _same(torch, d_out, x):
    return bool(torch.equal(d_out, torch.from_numpy(x).cuda()))


def _oracle_decode_all(blobs, ns):
    with cf.ThreadPoolExecutor(max_workers=min(len(blobs), os.cpu_count() or 1)) as ex:
        return list(ex.map(lambda bn: oracle.decode(*bn), zip(blobs, ns)))


def test_llama3_8b_layer_in_the_benchmark_launch(env):
    """The bench configuration: 7 projections, one batched launch; every
    tensor against its source and against the oracle's decode."""
    L, torch = env
    xs, blobs = _encode(L, synth.llama3_8b_layer().tensors)
    outs = _decode_batched(env, blobs)
    want = _oracle_decode_all(blobs, [x.size for x in xs])
    for x, w, o in zip(xs, want, outs):
        assert np.array_equal(w, x)
        assert _same(torch, o, x)
        assert np.array_equal(o.cpu().numpy(), w)


def test_alpha_sweep_points_full_size(env):
    """14336x4096 at alpha in {1.5,1.7,1.9,2.0} x max|w| in {448,112,28}:
    single-tensor decode; the most and least compressible points also
    against the oracle."""
    L, torch = env
    for a in synth.SWEEP_ALPHAS:
        for m in synth.SWEEP_MAXES:
            spec = synth.alpha_sweep_point(a, m).tensors[0]
            x = spec.generate()
            blob = L.encode(x)
            info = L.blob_info(blob)
            d_out = torch.empty(info.n, dtype=torch.uint8, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            L.decode(info, torch.from_numpy(blob).cuda(), d_out, status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0, (a, m)
            assert _same(torch, d_out, x), (a, m)
            if (a, m) in ((1.5, 28.0), (2.0, 448.0)):
                assert np.array_equal(d_out.cpu().numpy(), oracle.decode(blob, x.size)), (a, m)


@pytest.mark.slow
def test_moe_768_tensors_in_one_launch(env):
    """256 experts x {gate, up 2048x7168; down 7168x2048}, per-expert code
    books, one batched launch through the workspace descriptor table; every
    tensor checked by a 128-bit hash of its bytes, three also byte for byte
    against the source and the oracle."""
    L, torch = env
    specs = synth.moe_experts(256).tensors
    blobs, digests, sample = [], [], {}
    for i, t in enumerate(specs):
        x = t.generate()
        blobs.append(L.encode(x))
        digests.append(hashlib.blake2b(x.tobytes(), digest_size=16).digest())
        if i in (0, 383, 767):
            sample[i] = x
    assert L.batched_workspace_size(len(blobs)) > 0
    outs = _decode_batched(env, blobs)
    for i, o in enumerate(outs):
        got = o.cpu().numpy()
        assert hashlib.blake2b(got.tobytes(), digest_size=16).digest() == digests[i], i
        if i in sample:
            assert np.array_equal(got, sample[i])
            assert np.array_equal(got, oracle.decode(blobs[i], got.size))


@pytest.mark.slow
def test_llama3_70b_layers_into_one_reused_buffer(env):
    """Two Llama-3-70B layers (7 tensors each), decoded layer by layer into
    the same output buffers, each layer checked before the next overwrites it."""
    L, torch = env
    reuse = None
    for layer in range(2):
        specs = synth.llama3_70b_layer(layer).tensors
        xs, blobs = _encode(L, specs)
        if reuse is None:
            reuse = [torch.empty(x.size, dtype=torch.uint8, device="cuda") for x in xs]
        outs = _decode_batched(env, blobs, reuse_out=reuse)
        for x, o in zip(xs, outs):
            assert _same(torch, o, x), layer
        small = int(np.argmin([x.size for x in xs]))
        assert np.array_equal(outs[small].cpu().numpy(), oracle.decode(blobs[small], xs[small].size))
