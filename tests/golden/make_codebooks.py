"""Write the per-layer VQ3R (and VQ4P) codebooks of the synthetic workloads.

Page "3比特逼近4比特精度？WARP残差向量量化VQ3R的完整测量实验"
(xdnf.cn/news/289497), §2 and §4: codebooks are fitted per layer by Lloyd
k-means on vectors sampled from 12 experts, stage s on the residuals of
stage s-1.  The training itself is the oracle's (oracle.lloyd_train); this
script only draws the training vectors (seeded, synth) and writes the
result, which the CUDA path and the oracle then both take as input.

Workloads (synth/workloads.py):
  expert: the single expert (w1, w3, w2), 65536 vectors sampled uniformly
          without replacement from all of its vectors, 20 iterations;
  layer:  64 experts; 12 experts drawn, 65536 vectors from their matrices;
  sweep:  256 experts, Student-t(3) with outliers; same sampling;
  vq4p_layer: the layer workload's training vectors, VQ4P codebooks
          [4][64][8] (page §5) from oracle.vq4p_train, 20 iterations.
Training vectors are normalised by their row's FP16 scale first.

Usage: python tests/golden/make_codebooks.py [expert|layer|sweep|vq4p_layer ...]
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as wl  # noqa: E402

KINDS = (wl.W1, wl.W3, wl.W2)


def vectors_per_matrix(kind):
    rows, cols = wl.mat_shape(kind)
    return rows * (cols // 8)


def training_vectors(seed, dist, experts, n_vec):
    """Normalised training vectors (n_vec x 8), in draw order."""
    per_expert = sum(vectors_per_matrix(k) for k in KINDS)
    pool = len(experts) * per_expert
    pick = synth.sample(seed, wl.SAMPLE_VECTORS, pool, n_vec)
    e_slot, rem = np.divmod(pick, per_expert)
    kind_of = np.empty_like(pick)
    local = rem.copy()
    off = 0
    for k in KINDS:
        n = vectors_per_matrix(k)
        sel = (rem >= off) & (rem < off + n)
        kind_of[sel] = k
        local[sel] = rem[sel] - off
        off += n
    out = np.empty((n_vec, 8), dtype=np.float32)
    for slot, e in enumerate(experts):
        for k in KINDS:
            sel = np.nonzero((e_slot == slot) & (kind_of == k))[0]
            if len(sel) == 0:
                continue
            rows, cols = wl.mat_shape(k)
            V = cols // 8
            row, v = np.divmod(local[sel], V)
            urows, inv = np.unique(row, return_inverse=True)
            W = synth.fill_row_list(cols, urows, seed, wl.tag(int(e), k), dist, dtype="bf16")
            sc = oracle.row_scales(W, "bf16")
            r = oracle.normalize_rows(W, "bf16", sc).reshape(len(urows), V, 8)
            out[sel] = r[inv, v]
    return out


def make(name):
    if name == "expert":
        cfg, dist, experts = wl.EXPERT, wl.expert_dist(), [0]
    elif name in ("layer", "vq4p_layer"):
        cfg, dist = wl.LAYER, wl.expert_dist()
        experts = synth.sample(cfg["seed"], wl.SAMPLE_EXPERTS, cfg["experts"], cfg["train_experts"])
    elif name == "sweep":
        cfg, dist = wl.SWEEP, wl.sweep_dist()
        experts = synth.sample(cfg["seed"], wl.SAMPLE_EXPERTS, cfg["experts"], cfg["train_experts"])
    else:
        raise ValueError(name)
    vecs = training_vectors(cfg["seed"], dist, list(experts), cfg["train_vectors"])
    if name.startswith("vq4p_"):
        cb, trace = oracle.vq4p_train(vecs, cfg["lloyd_iters"])
    else:
        cb, trace = oracle.lloyd_train(vecs, cfg["lloyd_iters"])
    return cb, trace, list(int(e) for e in experts)


def shape(name):
    return (4, 64, 8) if name.startswith("vq4p_") else (3, 256, 8)


def path(name):
    return os.path.join(HERE, "codebooks_%s.txt" % name)


def write(name, cb, trace, experts):
    with open(path(name), "w") as f:
        S, K, _ = shape(name)
        fmt, fn = ("VQ4P", "oracle.vq4p_train") if S == 4 else ("VQ3R", "oracle.lloyd_train")
        f.write("# %s codebooks [%d][%d][8] float32 (hex bit patterns, one codeword per line)\n" % (fmt, S, K))
        f.write("# workload: %s; Lloyd on sampled normalised vectors (page §2, §4); experts %s\n" % (name, experts))
        f.write("# written by tests/golden/make_codebooks.py with %s only\n" % fn)
        f.write("# final training distortion per stage: %s\n" % " ".join("%.6e" % t for t in trace[:, -1]))
        u = cb.reshape(-1, 8).view(np.uint32)
        for row in u:
            f.write(" ".join("%08x" % int(w) for w in row) + "\n")


def load(name):
    rows = []
    with open(path(name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append([int(t, 16) for t in line.split()])
    return np.array(rows, dtype=np.uint32).view(np.float32).reshape(shape(name))


if __name__ == "__main__":
    for n in (sys.argv[1:] or ["expert", "layer", "sweep"]):
        cb, tr, ex = make(n)
        write(n, cb, tr, ex)
        print(n, "written; final distortion", tr[:, -1])
