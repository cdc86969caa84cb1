"""The seeded input generators shared by the oracle and the CUDA path (CPU):
deterministic, independent per stream and matrix, with the stated distributions
and the workloads' sizes."""
import numpy as np
import torch

from quantized_lora_fine_b200 import synth


def test_generators_are_deterministic_and_streams_independent():
    a = synth.normal_bf16((64, 128), 0.02, 0, synth.STREAM_W)
    b = synth.normal_bf16((64, 128), 0.02, 0, synth.STREAM_W)
    assert torch.equal(a, b)
    assert a.dtype == torch.bfloat16
    for other in (synth.normal_bf16((64, 128), 0.02, 1, synth.STREAM_W),          # another seed
                  synth.normal_bf16((64, 128), 0.02, 0, synth.STREAM_X),          # another stream
                  synth.normal_bf16((64, 128), 0.02, 0, synth.STREAM_W, 1)):      # another matrix
        assert not torch.equal(a, other)
    t1 = synth.student_t_bf16((32, 64), 5.0, 0.02, 0, synth.STREAM_W)
    assert torch.equal(t1, synth.student_t_bf16((32, 64), 5.0, 0.02, 0, synth.STREAM_W))


def test_stated_distributions():
    x = synth.normal_bf16((512, 1024), 0.02, 3, synth.STREAM_W).float().numpy()
    assert abs(x.mean()) < 3 * 0.02 / np.sqrt(x.size)
    assert abs(x.std() / 0.02 - 1) < 0.01
    # scale * t_nu: variance scale^2 nu / (nu - 2); heavier tails than a normal
    nu, sc = 5.0, 0.02
    t = synth.student_t_bf16((512, 1024), nu, sc, 4, synth.STREAM_W).float().numpy().astype(np.float64)
    assert abs(t.std() / (sc * np.sqrt(nu / (nu - 2))) - 1) < 0.03
    kurt = np.mean((t - t.mean()) ** 4) / t.var() ** 2
    assert kurt > 4.5            # a normal has 3; t_5 has 9 (sample estimates run lower)


def test_stack_draws_and_sizes():
    mats7 = synth.stack_matrices()
    assert len(mats7) == 224
    assert sum(m.out * m.inp for m in mats7) == 32 * (4 * 4096 * 4096 + 3 * 11008 * 4096)   # 6.48 G weights
    mats14 = synth.stack_matrices_14b()
    assert len(mats14) == 280
    assert sum(m.out * m.inp for m in mats14) == 12_687_769_600
    for m in mats7 + mats14:
        assert 3.0 <= m.nu <= 30.0 and 0.005 <= m.scale <= 0.05
    assert [m.index for m in mats7] == list(range(224))
    assert [(m.layer, m.name) for m in mats7[:8]] == [(0, "q"), (0, "k"), (0, "v"), (0, "o"), (0, "gate"),
                                                     (0, "up"), (0, "down"), (1, "q")]
    # each stack draws from its own seed, and a stack matrix's weights follow it
    assert all(m.seed == 0 for m in mats7) and all(m.seed == synth.STACK_14B_SEED for m in mats14)
    assert synth.STACK_14B_SEED != 0
    assert [(m.nu, m.scale) for m in mats7[:7]] != [(m.nu, m.scale) for m in mats14[:7]]
    small = synth.stack_matrices(n_layers=1, linears=(("a", 64, 128),), seed=synth.STACK_14B_SEED)[0]
    assert torch.equal(synth.stack_weight(small), synth.stack_weight(small, seed=synth.STACK_14B_SEED))
    assert not torch.equal(synth.stack_weight(small), synth.stack_weight(small, seed=0))


def test_bf16_bits_round_trip():
    t = synth.normal_bf16((17, 33), 1.0, 5, synth.STREAM_X)
    assert torch.equal(synth.from_bf16_bits(synth.bf16_bits(t)).reshape(t.shape), t)
