"""The seeded input recipe (no GPU): what the generators draw is what the
design states — deterministic per (seed, stream, index), outlier channels,
standard deviations, dtypes and the Wan2.2 token counts."""
import torch

from mxfp8_w8a8_quantized_b200 import synth


def test_streams_are_deterministic_and_distinct():
    a = synth.activations(64, 512, seed=3, index=1)
    assert torch.equal(a, synth.activations(64, 512, seed=3, index=1))
    assert not torch.equal(a, synth.activations(64, 512, seed=3, index=2))
    assert not torch.equal(a, synth.activations(64, 512, seed=4, index=1))
    w = synth.weights(32, 512, seed=3, index=1)
    assert torch.equal(w, synth.weights(32, 512, seed=3, index=1))
    assert a.dtype == torch.bfloat16 and w.dtype == torch.float32
    assert synth.bias(32, seed=3).dtype == torch.float16


def test_outlier_channels():
    K = 5120
    ch = synth.outlier_channels(K, seed=1)
    assert len(ch) == round(0.01 * K) == 51
    assert torch.equal(ch, torch.sort(ch).values) and len(set(ch.tolist())) == len(ch)
    assert int(ch.min()) >= 0 and int(ch.max()) < K
    x = synth.activations(4096, K, seed=1).float()
    std = x.std(dim=0)
    mask = torch.zeros(K, dtype=torch.bool)
    mask[ch] = True
    # outlier columns at about 20x the unit standard deviation of the rest
    assert 18.0 < float(std[mask].mean()) < 22.0
    assert 0.95 < float(std[~mask].mean()) < 1.05
    plain = synth.activations(4096, K, seed=1, outliers=False).float()
    assert 0.97 < float(plain.std()) < 1.03


def test_weight_and_bias_scales():
    for K in (512, 5120, 13824):
        w = synth.weights(256, K, seed=2)
        assert abs(float(w.std()) * K ** 0.5 - 1.0) < 0.02
        assert abs(float(w.mean())) < 0.01 / K ** 0.5 * 10
    b = synth.bias(20000, seed=2).float()
    assert abs(float(b.std()) - 0.01) < 0.0005


def test_token_counts_and_block_shapes():
    # 81 frames -> 21 latent frames; 16x spatial reduction
    assert synth.TOKENS_480P == 21 * (480 // 16) * (832 // 16) == 32760
    assert synth.TOKENS_832x1104 == 21 * (1104 // 16) * (832 // 16) == 75348
    lin = synth.block_linears()
    assert len(lin) == 10
    names = [n for n, *_ in lin]
    assert names.count("ffn.net.0.proj") == 1 and names.count("ffn.net.2") == 1
    shapes = {n: (K, N, kind) for n, K, N, kind in lin}
    assert shapes["ffn.net.0.proj"] == (synth.HIDDEN, synth.FFN, "video")
    assert shapes["ffn.net.2"] == (synth.FFN, synth.HIDDEN, "video")
    assert [n for n, *_, kind in lin if kind == "text"] == ["attn2.to_k", "attn2.to_v"]
    assert synth.WORKLOADS["c1_q_proj_480p"]["M"] == synth.TOKENS_480P
