"""Input recipes of the VQ3R workloads (shapes, distributions, seeds, tags).

The source pages measure on real expert weights of large MoE models
(xdnf.cn/news/289497, §3.1-§3.3), which are not available here; these seeded
synthetic tensors stand in for them, with DeepSeek-style expert shapes
(gate/up 2048 x 7168, down 7168 x 2048).

Tags: tensor tag = expert * 8 + kind, kind 0 = w1 (gate), 1 = w3 (up),
2 = w2 (down), 3 = token activations for gate/up, 4 = per-expert inputs of
the down projection.  Sampling streams use SAMPLE_EXPERTS / SAMPLE_VECTORS.
"""
import synth

W1, W3, W2, X_GATEUP, X_DOWN = 0, 1, 2, 3, 4
HIDDEN, INTER = 7168, 2048
SAMPLE_EXPERTS = 0xF00001
SAMPLE_VECTORS = 0xF00002
TINY_SEED, EXPERT_SEED, LAYER_SEED, ACT_SEED, SWEEP_SEED = 0, 1, 2, 3, 4


def tag(expert, kind):
    return expert * 8 + kind


def mat_shape(kind):
    """(rows, cols) of an expert matrix: w1/w3 map hidden -> inter, w2 inter -> hidden."""
    return (INTER, HIDDEN) if kind in (W1, W3) else (HIDDEN, INTER)


def expert_dist():
    """Student-t(4) times a per-row log-normal(0, 0.5) factor."""
    return synth.student_t(4, row_sigma=0.5)


def sweep_dist():
    """Student-t(3), log-normal(0, 0.5) rows, 0.1% outliers at +-20 sigma (sigma = sqrt(3))."""
    return synth.student_t(3, row_sigma=0.5, outlier_p=1e-3, outlier_mag=20.0 * 3.0 ** 0.5)


TINY = dict(name="tiny-256x512-f32", rows=256, cols=512, seed=TINY_SEED, dtype="f32", lloyd_iters=10)
EXPERT = dict(name="expert-2048x7168+7168x2048-bf16", experts=1, seed=EXPERT_SEED, dtype="bf16",
              train_vectors=65536, lloyd_iters=20)
LAYER = dict(name="moe-layer-64x3-bf16", experts=64, seed=LAYER_SEED, dtype="bf16", train_experts=12,
             train_vectors=65536, lloyd_iters=20)
SWEEP = dict(name="moe-sweep-256x3-bf16-t3-outliers", experts=256, seed=SWEEP_SEED, dtype="bf16",
             train_experts=12, train_vectors=65536, lloyd_iters=20)
DECODE_STEP = dict(name="moe-decode-step-8-experts", experts=8, batches=(1, 4, 8, 32), act_seed=ACT_SEED)
