"""The seeded input generator: determinism, counter addressing, ranges and moments."""
import numpy as np

import synth


def test_counter_addressing_is_slice_consistent():
    a = synth.words(3, 77, 0, 1000)
    assert np.array_equal(a[100:300], synth.words(3, 77, 100, 200))
    b = synth.uniform_bytes(3, 77, 0, 4000)
    assert np.array_equal(b[:8], a[0:1].view(np.uint8))
    assert np.array_equal(b[1234:2345], synth.uniform_bytes(3, 77, 1234, 1111))
    c = synth.codes_i8(3, 78, 0, 5000)
    assert np.array_equal(c[777:999], synth.codes_i8(3, 78, 777, 222))
    assert not np.array_equal(synth.words(3, 77, 0, 8), synth.words(4, 77, 0, 8))
    assert not np.array_equal(synth.words(3, 77, 0, 8), synth.words(3, 79, 0, 8))


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0 produces, as its first three outputs, mix(0),
    # mix(gamma), mix(2*gamma) in the additive form used here; these are the
    # published first outputs of SplittableRandom-style splitmix64 from state 0.
    gamma = 0x9E3779B97F4A7C15

    def mix(z):
        z = (z + gamma) & (2 ** 64 - 1)
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2 ** 64 - 1)
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2 ** 64 - 1)
        return z ^ (z >> 31)

    assert mix(0) == 0xE220A8397B1DCDAF
    assert mix(gamma) == 0x6E789E6AA1B965F4
    key = mix(mix(5) ^ 9)
    want = [mix((key + i) & (2 ** 64 - 1)) for i in range(4)]
    assert synth.words(5, 9, 0, 4).tolist() == want


def test_code_ranges_and_scale_range():
    sh = synth.CONFIGS["tiny"]
    for q, lo, hi in [(4, -8, 7), (2, -2, 1)]:
        codes, sc = synth.expert_matrix(sh.with_(qtype=q), 0, 1, synth.DOWN)
        assert codes.shape == (sh.H, sh.I * q // 8)
        assert np.all((sc >= 0.01) & (sc < 0.05))
    c8, _ = synth.expert_matrix(sh.with_(qtype=8), 0, 1, synth.GATE)
    v = c8.view(np.int8)
    assert v.min() == -127 and v.max() == 127
    counts = np.bincount(v.astype(np.int64).reshape(-1) + 127, minlength=255)
    assert counts.min() > 0.5 * counts.mean()


def test_normal_moments_and_bf16():
    z = synth.normals(0, 5, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    sh = synth.CONFIGS["decode"]
    W = synth.router_weight(sh.with_(E=16))
    assert W.dtype == np.float32 and abs(W.std() - 0.02) < 0.001
    x = synth.hidden_states(sh.with_(T=3))
    assert x.dtype == np.uint16 and x.shape == (3, 6144)
    # token rows do not depend on how many tokens are drawn
    assert np.array_equal(x[2], synth.hidden_states(sh, tokens=[2])[0])


def test_verify_inputs_are_correlated_and_prefill_bias_is_skewed():
    sh = synth.CONFIGS["verify"]
    x = synth.bf16_to_f32(synth.hidden_states(sh)).astype(np.float64)
    c = np.corrcoef(x)
    assert np.all(c[np.triu_indices(4, 1)] > 0.7)
    b = synth.router_bias(synth.CONFIGS["prefill"])
    r = synth.zipf_ranks(synth.CONFIGS["prefill"])
    assert sorted(r.tolist()) == list(range(1, 257))
    assert np.corrcoef(np.log(r), b)[0, 1] < -0.5
