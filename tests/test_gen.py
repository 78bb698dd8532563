"""The seeded input generator: formats, determinism, range independence and
the workloads' value distributions and structure."""
import numpy as np
import torch

import gen


def test_e4m3_encoding_of_small_integers_is_exact():
    v = np.arange(-16, 17, dtype=np.float64)
    b = gen.encode_e4m3(v)
    dec = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(dec, v)


def test_bf16_encoding_matches_library_rounding():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(10000) * 3
    ref = torch.from_numpy(v).float().bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gen.encode_bf16(v), ref)


def test_subranges_equal_slices_and_threads_do_not_matter():
    full = gen.int_e4m3(5, 1, 0, 100000, -8, 8, nthreads=1)
    part = gen.int_e4m3(5, 1, 31337, 20000, -8, 8, nthreads=4)
    assert np.array_equal(full[31337:51337], part)
    n1 = gen.normal_bf16(5, 4, 0, 50001, nthreads=1)
    n2 = gen.normal_bf16(5, 4, 777, 1001, nthreads=3)
    assert np.array_equal(n1[777:1778], n2)
    assert not np.array_equal(gen.int_e4m3(6, 1, 0, 1000), gen.int_e4m3(5, 1, 0, 1000))


def test_iid_distributions():
    ints = torch.from_numpy(gen.int_e4m3(1, 1, 0, 170000)).view(torch.float8_e4m3fn).float().numpy()
    ints = ints.astype(np.int64)
    vals, cnt = np.unique(ints, return_counts=True)
    assert vals.tolist() == list(range(-8, 9))
    assert cnt.min() > 0.9 * 10000 and cnt.max() < 1.1 * 10000
    w = gen.int_f32(1, 3, 0, 40000, 0, 3)
    assert set(np.unique(w).tolist()) == {0.0, 1.0, 2.0, 3.0}
    z = torch.from_numpy(gen.normal_bf16(1, 4, 0, 200000).view(np.int16)).view(
        torch.bfloat16).double().numpy()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_workload_shapes():
    c1 = gen.TINY_PREFILL
    inp = gen.prefill_inputs(c1)
    assert inp["q_I"].shape == (2048, 4, 64) and inp["k_I"].shape == (2048, 64)
    assert inp["w"].shape == (2048, 4) and inp["Q"].shape == (2048, 8, 64)
    assert inp["K"].shape == (2048, 2, 64) and inp["V"].shape == (2048, 2, 64)
    c4 = gen.DECODE_B64
    n = gen.decode_lengths(c4)
    assert n.shape == (64,) and n.min() >= 32768 and n.max() <= 262144
    off = gen.decode_offsets(c4)
    assert off[0] == 0 and np.all(np.diff(off) == n)


def test_video_structure():
    c5 = gen.VIDEO_256K
    assert c5.frames * (c5.frame_text + c5.frame_vision) + 64 == c5.L
    ft = c5.frame_text + c5.frame_vision
    # three frames' worth of indexer keys
    kI = torch.from_numpy(gen.prefill_kI(c5, 0, 3 * ft)).view(torch.float8_e4m3fn).float().numpy()
    kI = kI.astype(np.int64)
    assert kI.min() >= -8 and kI.max() <= 8
    for f in range(3):
        vis = kI[f * ft + c5.frame_text:(f + 1) * ft]
        cen = np.round(vis.mean(axis=0))
        # vision tokens stay within +-2 of the frame centroid (in [-6, 6])
        assert np.all(np.abs(vis - cen) <= 3) and np.all(np.abs(cen) <= 6)
        txt = kI[f * ft:f * ft + c5.frame_text]
        assert np.abs(txt - cen).max() > 2  # text tokens are not clustered
    # the trailing 64 tokens are text
    tail = gen.prefill_kI(c5, c5.L - 64, c5.L)
    assert tail.shape == (64, 128)
    # queries of a vision token share their frame's centroid with the keys
    q = torch.from_numpy(gen.prefill_qI(c5, ft + 100, ft + 101)).view(
        torch.float8_e4m3fn).float().numpy().astype(np.int64)[0]
    kv = kI[ft + c5.frame_text:2 * ft]
    assert np.all(np.abs(q - np.round(kv.mean(axis=0))) <= 3)
    # K/V: vision tokens = centroid + N(0, 0.5^2)
    K = torch.from_numpy(gen.prefill_K(c5, 0, ft).view(np.int16)).view(
        torch.bfloat16).double().numpy()
    vis = K[c5.frame_text:]
    assert abs(vis.std(axis=0).mean() - 0.5) < 0.03
