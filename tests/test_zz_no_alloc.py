"""ecf8_decode_batched_noalloc against ecf8_decode_batched, on the GPU.

The no-allocation call is for code that cannot allocate device memory at the
moment it decodes weights: a plugin inside an inference engine that owns all
device memory and gives the plugin no scratch space, or a serving loop that
must not call cudaMalloc because that call synchronises the whole device.
Instead of a caller workspace it keeps the per-call descriptor table in device
memory the library holds for the life of the process.

Both tests go through the C ABI (ctypes binding) and compare bytes exactly,
as every decode test here does.  Two calls are made back to back with
different tensor sets: every call shares the library's one table, so the
second call must fully replace what the first left there.
"""
import numpy as np
import pytest

import ecf8_synth as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env(gpu_available):
    import torch
    import lossless_fp8_weight_b200 as L
    return L, torch


def _tensor_set(L, count, seed):
    r = np.random.default_rng(seed)
    spec = synth.alpha_sweep_point(1.7, 448.0).tensors[0]
    xs = [spec.generate(begin=int(r.integers(0, 1 << 24)), count=int(r.integers(1, 300_000))) for _ in range(count)]
    blobs = [L.encode(x) for x in xs]
    return xs, blobs


def _decode_both(L, torch, xs, blobs):
    infos = [L.blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).cuda() for b in blobs]
    ref_out = [torch.full((i.n,), 0xA5, dtype=torch.uint8, device="cuda") for i in infos]
    new_out = [torch.full((i.n,), 0x5A, dtype=torch.uint8, device="cuda") for i in infos]
    ws = torch.empty(max(L.batched_workspace_size(len(blobs)), 16), dtype=torch.uint8, device="cuda")
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_new = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.decode_batched([L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, ref_out)], workspace=ws,
                     status=st_ref)
    before = L.launch_count()
    L.decode_batched_noalloc([L.BatchItem(i, b, o) for i, b, o in zip(infos, d_blobs, new_out)], status=st_new)
    assert L.launch_count() == before + 1
    torch.cuda.synchronize()
    assert int(st_ref.item()) == 0 and int(st_new.item()) == 0
    for x, a, b in zip(xs, ref_out, new_out):
        a, b = a.cpu().numpy(), b.cpu().numpy()
        assert np.array_equal(a, b)
        assert np.array_equal(b, x)


def test_noalloc_equals_batched_on_two_calls_in_a_row(env):
    L, torch = env
    xs1, blobs1 = _tensor_set(L, 100, seed=1)  # past the inline limit: decode_batched uses its workspace
    xs2, blobs2 = _tensor_set(L, 7, seed=2)    # a smaller, different set overwrites part of the table
    _decode_both(L, torch, xs1, blobs1)
    _decode_both(L, torch, xs2, blobs2)


def test_noalloc_rejects_more_tensors_than_its_table(env):
    L, torch = env
    x = np.full(64, 0x38, np.uint8)
    blob = L.encode(x)
    info = L.blob_info(blob)
    d_blob = torch.from_numpy(blob).cuda()
    out = torch.empty(64, dtype=torch.uint8, device="cuda")
    items = [L.BatchItem(info, d_blob, out)] * (L.NOALLOC_MAX_TENSORS + 1)
    before = L.launch_count()
    with pytest.raises(L.Ecf8Error) as e:
        L.decode_batched_noalloc(items)
    assert e.value.code == -9
    assert L.launch_count() == before


def test_noalloc_fills_its_table_to_the_last_entry(env):
    """Exactly ECF8_NOALLOC_MAX_TENSORS tensors: every slot of the library's
    table is written and read, the last one included."""
    L, torch = env
    r = np.random.default_rng(5)
    spec = synth.single_normal_1k().tensors[0]
    xs = [spec.generate(begin=int(r.integers(0, 1 << 20)), count=int(r.integers(1, 600)))
          for _ in range(L.NOALLOC_MAX_TENSORS)]
    _decode_both(L, torch, xs, [L.encode(x) for x in xs])
