"""The seeded input generator: deterministic, thread-count independent, right shapes."""
import os
import subprocess
import sys

import numpy as np

import synth


def test_deterministic_and_offset_consistent():
    a = synth.normal_f32(10000, seed=3, stream=1)
    b = synth.normal_f32(10000, seed=3, stream=1)
    assert (a == b).all()
    tail = synth.normal_f32(5000, seed=3, stream=1, offset=5000)
    assert (a[5000:] == tail).all()
    assert not (synth.normal_f32(100, seed=4, stream=1) == a[:100]).all()
    assert not (synth.normal_f32(100, seed=3, stream=2) == a[:100]).all()


def test_thread_count_independent():
    code = "import synth,sys; sys.stdout.write(synth.latent_weights(64, 640, seed=9).tobytes().hex()[:4000])"
    outs = []
    for threads in ("1", "4"):
        env = dict(os.environ, OMP_NUM_THREADS=threads)
        outs.append(subprocess.check_output([sys.executable, "-c", code], env=env,
                                            cwd=os.path.dirname(os.path.dirname(__file__))))
    assert outs[0] == outs[1]


def test_distributions():
    w = synth.latent_weights(512, 2048, seed=0)
    assert abs(w.std() - 0.02) < 2e-4 and abs(w.mean()) < 2e-4
    x = synth.activations_f32(8, 2560, seed=1)
    ch = synth.outlier_channels(2560, seed=1)
    assert len(ch) == 26 and len(set(ch.tolist())) == 26
    mask = np.zeros(2560, bool)
    mask[ch] = True
    assert 15 < x[:, mask].std() < 25 and 0.9 < x[:, ~mask].std() < 1.1
    assert [synth.outlier_count(k) for k in (2560, 3200, 8640, 8192, 28672)] == [26, 32, 86, 82, 287]


def test_bf16_round_trip():
    x = synth.activations_f32(4, 256, seed=5)
    bits = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits)
    assert np.abs(back - x).max() <= np.abs(x).max() * 2 ** -8
    assert (synth.f32_to_bf16_bits(back) == bits).all()
