"""Seeded synthetic workloads: parameter-tensor lists and input generators.

Holds none of the method's arithmetic: only the shapes of the model families
the workloads are named after, the seeds, and random draws. Both the CUDA
path and the CPU oracle consume the bytes these functions produce.

Workloads (the step's inputs are gradients of these parameter lists):
  tiny      4 tensors [1024x512, 512, 512x1000, 1000], R=4, bf16 grads
            ~N(0, 1e-3), static loss scale 1.0, 10 steps, one bucket.
  gpt2s     GPT-2-small-shaped list (12 layers, d=768, 4d MLP, vocab 50257,
            ctx 1024, tied head; 124,439,808 params, 148 tensors), R=8, fp16
            grads ~N(0, 1e-4) times the loss scale, dynamic scaling from 2^16
            growing every 100 clean steps, +inf injected at step 3 (replica 0,
            tensor 74, element 0), 25M-element buckets.
  d1p3b     1.3B decoder-shaped list (24 layers, d=2048, 4d MLP, vocab 50257,
            learned positions for ctx 2048, tied head; 292 tensors), R=8, bf16
            grads ~N(0, 1e-4), no loss scaling, 5 steps, per-layer gather.
  llama3b   Llama-style 3B-shaped list (28 layers, d=3072, SwiGLU ffn 8192,
            24 q / 8 kv heads of 128, vocab 128256, untied embeddings; 255
            tensors), R=4, bf16 grads 1e-4 * Student-t(3), 3 steps, 50M buckets.
  irr_r16 / irr_r2
            10,000 tensors with sizes round(exp(U(0, ln 4M))) clamped to
            [1, 4M] (4M = 2^22), fp16 grads, dynamic scaling; R=2 on the list
            as drawn (about 2.75B params expected), R=16 on the same sizes
            rescaled to 256M in total. The last size gets +1 if the total is
            divisible by R. 100 tensors per layer.
"""
import math

import numpy as np
import torch

BF16, FP16 = 0, 1
NONE, STATIC, DYNAMIC = 0, 1, 2
TORCH_HALF = {BF16: torch.bfloat16, FP16: torch.float16}
MASTER_SIGMA = 0.02


# ---- parameter lists -------------------------------------------------------

def gpt_tensors(d, n_layers, vocab, ctx, ffn):
    """GPT-2-style decoder with learned positions and a tied head.
    Returns (names, numels, layer_ids): layer 0 = embeddings, 1..n = blocks,
    n+1 = final LayerNorm."""
    names, numels, layers = [], [], []

    def add(name, n, layer):
        names.append(name)
        numels.append(int(n))
        layers.append(layer)

    add("wte", vocab * d, 0)
    add("wpe", ctx * d, 0)
    for i in range(n_layers):
        L = i + 1
        p = f"h{i}."
        add(p + "ln_1.w", d, L)
        add(p + "ln_1.b", d, L)
        add(p + "attn.c_attn.w", d * 3 * d, L)
        add(p + "attn.c_attn.b", 3 * d, L)
        add(p + "attn.c_proj.w", d * d, L)
        add(p + "attn.c_proj.b", d, L)
        add(p + "ln_2.w", d, L)
        add(p + "ln_2.b", d, L)
        add(p + "mlp.c_fc.w", d * ffn, L)
        add(p + "mlp.c_fc.b", ffn, L)
        add(p + "mlp.c_proj.w", ffn * d, L)
        add(p + "mlp.c_proj.b", d, L)
    add("ln_f.w", d, n_layers + 1)
    add("ln_f.b", d, n_layers + 1)
    return names, numels, layers


def llama_tensors(d, n_layers, vocab, ffn, n_q, n_kv, head_dim):
    """Llama-style decoder, RMSNorm, SwiGLU, GQA, untied embeddings.
    Layer 0 = embedding, 1..n = blocks, n+1 = final norm + lm_head."""
    names, numels, layers = [], [], []

    def add(name, n, layer):
        names.append(name)
        numels.append(int(n))
        layers.append(layer)

    add("embed", vocab * d, 0)
    for i in range(n_layers):
        L = i + 1
        p = f"l{i}."
        add(p + "attn_norm", d, L)
        add(p + "q", d * n_q * head_dim, L)
        add(p + "k", d * n_kv * head_dim, L)
        add(p + "v", d * n_kv * head_dim, L)
        add(p + "o", n_q * head_dim * d, L)
        add(p + "mlp_norm", d, L)
        add(p + "gate", d * ffn, L)
        add(p + "up", d * ffn, L)
        add(p + "down", ffn * d, L)
    add("final_norm", d, n_layers + 1)
    add("lm_head", vocab * d, n_layers + 1)
    return names, numels, layers


def irregular_sizes(n=10_000, max_size=1 << 22, seed=1238):
    rng = np.random.default_rng(seed)
    u = rng.uniform(0.0, math.log(max_size), n)
    return np.clip(np.rint(np.exp(u)), 1, max_size).astype(np.int64)


def irregular_tensors(R, total=None, seed=1238):
    sizes = irregular_sizes(seed=seed)
    if total is not None:
        sizes = np.maximum(1, np.rint(sizes * (total / sizes.sum()))).astype(np.int64)
    if int(sizes.sum()) % R == 0:
        sizes[-1] += 1
    numels = sizes.tolist()
    names = [f"t{k}" for k in range(len(numels))]
    layers = [k // 100 for k in range(len(numels))]
    return names, numels, layers


def workload(name):
    """The named workload as a dict (see the module docstring)."""
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    if name == "tiny":
        names = ["w1", "b1", "w2", "b2"]
        numels = [1024 * 512, 512, 512 * 1000, 1000]
        return dict(name=name, index=0, names=names, numels=numels, layer_ids=[0, 0, 1, 1],
                    R=4, dtype=BF16, dist="normal", sigma=1e-3, mode=STATIC, init_scale=1.0,
                    interval=1000, steps=10, bucket_elems=0, inject=None, hp=hp)
    if name == "gpt2s":
        names, numels, layers = gpt_tensors(768, 12, 50257, 1024, 3072)
        return dict(name=name, index=1, names=names, numels=numels, layer_ids=layers, R=8,
                    dtype=FP16, dist="normal", sigma=1e-4, mode=DYNAMIC, init_scale=2.0 ** 16,
                    interval=100, steps=10, bucket_elems=25_000_000,
                    inject=dict(step=3, rank=0, tensor=74, element=0), hp=hp)
    if name == "d1p3b":
        names, numels, layers = gpt_tensors(2048, 24, 50257, 2048, 8192)
        return dict(name=name, index=2, names=names, numels=numels, layer_ids=layers, R=8,
                    dtype=BF16, dist="normal", sigma=1e-4, mode=NONE, init_scale=1.0,
                    interval=1000, steps=5, bucket_elems=0, inject=None, hp=hp)
    if name == "llama3b":
        names, numels, layers = llama_tensors(3072, 28, 128256, 8192, 24, 8, 128)
        return dict(name=name, index=3, names=names, numels=numels, layer_ids=layers, R=4,
                    dtype=BF16, dist="t3", sigma=1e-4, mode=NONE, init_scale=1.0,
                    interval=1000, steps=3, bucket_elems=50_000_000, inject=None, hp=hp)
    if name in ("irr_r16", "irr_r2"):
        R = 16 if name == "irr_r16" else 2
        names, numels, layers = irregular_tensors(R, total=256_000_000 if R == 16 else None)
        return dict(name=name, index=4, names=names, numels=numels, layer_ids=layers, R=R,
                    dtype=FP16, dist="normal", sigma=1e-4, mode=DYNAMIC, init_scale=2.0 ** 16,
                    interval=100, steps=3, bucket_elems=25_000_000, inject=None, hp=hp)
    raise KeyError(name)


WORKLOADS = ("tiny", "gpt2s", "d1p3b", "llama3b", "irr_r16", "irr_r2")


# ---- seeded draws ----------------------------------------------------------

def _gen(device, *key):
    g = torch.Generator(device=device)
    s = 1234
    for k in key:
        s = (s * 1_000_003 + int(k) + 7) % (2 ** 61 - 1)
    g.manual_seed(s)
    return g


def _draw(n, dist, gen, device):
    if dist == "normal":
        return torch.randn(n, generator=gen, device=device, dtype=torch.float32)
    if dist == "t3":
        # Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3)
        z = torch.randn(n, generator=gen, device=device, dtype=torch.float32)
        c = torch.randn(3, n, generator=gen, device=device, dtype=torch.float32)
        chi2 = (c * c).sum(0)
        return z / torch.sqrt(chi2 / 3.0)
    raise KeyError(dist)


def tensor_grads(numel, dist, sigma, scale, dtype, seed, step, rank, k, device):
    """Gradient replica `rank` of tensor k at `step`, as the half values a
    backward pass with loss scale `scale` would hold: half(scale * sigma * x)."""
    x = _draw(numel, dist, _gen(device, seed, 1, step, rank, k), device)
    return (x * sigma * scale).to(TORCH_HALF[dtype])


def tensor_master(numel, seed, k, device):
    """Initial fp32 master weights of tensor k: N(0, 0.02)."""
    return torch.randn(numel, generator=_gen(device, seed, 2, k), device=device,
                       dtype=torch.float32) * MASTER_SIGMA


def flat_grads(wl, step, rank, scale, device, seed=None):
    """Unpadded gradient replica (all tensors concatenated), half dtype."""
    seed = wl["index"] if seed is None else seed
    return torch.cat([tensor_grads(n, wl["dist"], wl["sigma"], scale, wl["dtype"], seed, step,
                                   rank, k, device) for k, n in enumerate(wl["numels"])])


def flat_master(wl, device, seed=None):
    seed = wl["index"] if seed is None else seed
    return torch.cat([tensor_master(n, seed, k, device) for k, n in enumerate(wl["numels"])])


def custom_workload(numels, R, dtype, mode=NONE, init_scale=1.0, interval=1000,
                    sigma=1e-3, dist="normal", layer_ids=None, bucket_elems=0, index=99):
    """A small workload with a caller-given tensor list (for parity tests)."""
    return dict(name="custom", index=index, names=[f"t{k}" for k in range(len(numels))],
                numels=[int(n) for n in numels], layer_ids=layer_ids, R=R, dtype=dtype,
                dist=dist, sigma=sigma, mode=mode, init_scale=init_scale, interval=interval,
                steps=1, bucket_elems=bucket_elems, inject=None,
                hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01))
