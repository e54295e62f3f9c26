"""The seeded input generator: determinism, stream independence, the stated
distributions, the Zipf trace, and (on a GPU) byte-identity of the device
build with the host build."""
import numpy as np
import pytest

import synth


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0 yields, as its first outputs, the published
    # sequence of the generator (Steele, Lea, Flood 2014; the same values
    # java.util.SplittableRandom and the reference C code of Vigna print).
    assert synth.draw(0, 0) == 0xE220A8397B1DCDAF
    assert synth.draw(0, 1) == 0x6E789E6AA1B965F4
    assert synth.draw(0, 2) == 0x06C45D188009454F


def test_deterministic_and_distinct_streams():
    a = synth.expert(synth.TINY, 0, 0, 3)
    b = synth.expert(synth.TINY, 0, 0, 3)
    c = synth.expert(synth.TINY, 0, 0, 4)
    d = synth.expert(synth.TINY, 1, 0, 3)
    for k in a:
        assert np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])
        assert not np.array_equal(a[k], d[k])
    x1 = synth.tokens(synth.TINY, 0, 5, 2)
    x2 = synth.tokens(synth.TINY, 0, 6, 1)
    assert np.array_equal(x1[1], x2[0])


def test_distributions():
    sh = synth.GLM
    e = synth.expert(sh, 0, 0, 0)
    q = e["q_gate"]
    nib = np.concatenate([q & 0xF, q >> 4]).ravel()
    counts = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(counts - 1 / 16) < 0.002)
    s = e["s_gate"].view(np.float16).astype(np.float64)
    assert s.min() >= 0.005 - 1e-5 and s.max() <= 0.02 + 1e-5
    assert abs(s.mean() - 0.0125) < 2e-4
    w, b = synth.router(sh, 0, 0)
    assert abs(w.std() - 0.02) < 2e-4 and abs(w.mean()) < 1e-4
    assert b.min() >= -0.1 and b.max() <= 0.1
    x = synth.bf16_to_f32(synth.tokens(sh, 0, 0, 16))
    assert abs(x.std() - 1.0) < 0.02


def test_zipf_trace_properties():
    tr = synth.zipf_trace(0, 2, 256, 8, 4000)
    assert tr.shape == (4000, 2, 8)
    assert np.all(np.diff(tr, axis=2) > 0)
    assert tr.min() >= 0 and tr.max() < 256
    # the most popular expert of a layer is picked far more often than the
    # median one, and the two layers use different permutations
    c0 = np.bincount(tr[:, 0].ravel(), minlength=256)
    c1 = np.bincount(tr[:, 1].ravel(), minlength=256)
    assert c0.max() > 20 * np.median(c0)
    assert np.argmax(c0) != np.argmax(c1) or not np.array_equal(np.argsort(c0), np.argsort(c1))
    assert np.array_equal(tr, synth.zipf_trace(0, 2, 256, 8, 4000))


def test_correlated_tokens_overlap():
    sh = synth.GLM
    x = synth.bf16_to_f32(synth.correlated_tokens(sh, 0, 4)).astype(np.float64)
    x0 = synth.bf16_to_f32(synth.tokens(sh, 0, 0, 1)[0]).astype(np.float64)
    for t in range(4):
        d = x[t] - x0
        assert 0.03 < d.std() < 0.07


@pytest.mark.gpu
def test_device_generator_matches_host():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sh = synth.GLM
    ptrs, bufs = {}, {}
    for name, dt, shp, tag in synth.expert_layout(sh):
        t = torch.empty(int(np.prod(shp)) * np.dtype(dt).itemsize, dtype=torch.uint8, device="cuda")
        bufs[name] = t
        ptrs[name] = t.data_ptr()
    synth.fill_expert_device(sh, 0, 2, 17, ptrs, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    host = synth.expert(sh, 0, 2, 17)
    for name, dt, shp, tag in synth.expert_layout(sh):
        dev = bufs[name].cpu().numpy().view(dt).reshape(shp)
        assert np.array_equal(dev, host[name]), name


def test_expert_into_matches_expert():
    # the in-place generator (pinned host stores) gives the same tensors
    buf = np.zeros(synth.expert_stride(synth.TINY), dtype=np.uint8)
    offs = synth.expert_into(synth.TINY, 0, 2, 5, buf.ctypes.data)
    for name, a in synth.expert(synth.TINY, 0, 2, 5).items():
        got = buf[offs[name]:offs[name] + a.nbytes].view(a.dtype).reshape(a.shape)
        assert np.array_equal(got, a), name
