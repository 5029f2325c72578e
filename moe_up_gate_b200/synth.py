"""Seeded synthetic inputs for the Q8_0 decode and MoE up/gate workloads.

This module only draws numbers: weights, activations, routing ids and routing
weights.  It holds none of the method's arithmetic (no quantization, no dot
products, no SwiGLU, no combine) and is the one module that the CPU oracle
side and the CUDA side both use, so that both see the same inputs.

Recipe (every tensor gets its own generator):
  * seed = 1000 * c + 10 * l + j for workload c, layer l, tensor j;
  * ``torch.Generator(device).manual_seed(seed)``; the values depend on the
    device the generator runs on, so a test or a benchmark draws each tensor
    once and hands the same tensor to both sides;
  * weights: ``randn * 0.02`` (fp32), later quantized to Q8_0 by each side;
  * activations x: ``randn`` (N(0, 1)), or ``randn * 0.02`` in the 30-layer
    MoE sweep where every tensor is N(0, 0.02);
  * routing ids per token: the first ``n_used`` entries of a uniformly random
    permutation of the experts (``argsort`` of uniform draws), so the ids of a
    token are distinct and uniform;
  * routing weights: softmax over ``n_used`` N(0, 1) logits, computed in fp64
    and stored as fp32 (the router is outside the path; these are inputs).

Workload shapes (the Q8_0 decode matvec set follows the Llama 2 110M
(stories110M) decode of the "narray-llm" README; the MoE shapes follow the
Gemma 4 26B-A4B MoE layer of the news.hada.io article: 30 layers, 8 active
experts per token):
  1  GEMV 768 x 768, batch 1
  2  Llama-2-110M-shaped matvec set: 12 layers x {wq, wk, wv, wo 768x768,
     w1, w3 2048x768, w2 768x2048} + classifier 32000x768, batch 1
  3  dense up_gate [4096 -> 2*14336] + down [14336 -> 4096], 1 and 8 tokens
  4  MoE layer: n_embd 2816, n_ff 704, 128 experts, top-8, 1 and 16 tokens
  5  30 MoE layers of workload 4's shape, 1/4/16/64/256 tokens
  (and the feed-forward layers of workload 2 with separate gate (w1) and up
  (w3) weights packed into one combined up/gate tensor: llama_ffn_tensors)
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

W_STD = 0.02


def seed_of(c: int, layer: int, j: int) -> int:
    return 1000 * c + 10 * layer + j


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """fp32 N(0, std^2) tensor of the given shape, drawn on ``device``."""
    g = _gen(seed, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def routing_ids(n_tok: int, n_exp: int, n_used: int, seed: int) -> torch.Tensor:
    """int32 [n_tok, n_used]: per token, n_used distinct experts, uniform (CPU)."""
    g = _gen(seed, "cpu")
    u = torch.rand((n_tok, n_exp), generator=g, dtype=torch.float64)
    return u.argsort(dim=1)[:, :n_used].to(torch.int32).contiguous()


def routing_weights(n_tok: int, n_used: int, seed: int) -> torch.Tensor:
    """fp32 [n_tok, n_used]: softmax over n_used N(0, 1) logits per token (CPU)."""
    g = _gen(seed, "cpu")
    logits = torch.randn((n_tok, n_used), generator=g, dtype=torch.float64)
    return torch.softmax(logits, dim=1).to(torch.float32).contiguous()


# --------------------------------------------------------------------------
# workload shapes
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class MoeShape:
    n_embd: int
    n_ff: int
    n_exp: int
    n_used: int


DENSE_FFN = MoeShape(n_embd=4096, n_ff=14336, n_exp=1, n_used=1)
MOE_LAYER = MoeShape(n_embd=2816, n_ff=704, n_exp=128, n_used=8)
MOE_LAYERS = 30
MOE_SWEEP_TOKENS = (1, 4, 16, 64, 256)

LLAMA_DIM = 768
LLAMA_HIDDEN = 2048
LLAMA_LAYERS = 12
LLAMA_VOCAB = 32000


def llama_matvec_set():
    """[(name, rows, k)] of the 85 matvecs of one Llama-2-110M-shaped decode step, in model order."""
    out = []
    d, hdim = LLAMA_DIM, LLAMA_HIDDEN
    for layer in range(LLAMA_LAYERS):
        for name, rows, k in (("wq", d, d), ("wk", d, d), ("wv", d, d), ("wo", d, d),
                              ("w1", hdim, d), ("w3", hdim, d), ("w2", d, hdim)):
            out.append((f"l{layer}.{name}", rows, k))
    out.append(("classifier", LLAMA_VOCAB, d))
    return out


LLAMA_FFN = MoeShape(n_embd=LLAMA_DIM, n_ff=LLAMA_HIDDEN, n_exp=1, n_used=1)


def llama_ffn_tensors(layer: int, n_tok: int, device="cpu"):
    """fp32 tensors of one Llama-2-110M-shaped feed-forward layer with separate
    gate and up weights: w1 (gate) and w3 (up) [2048, 768], w2 (down)
    [768, 2048], x [n_tok, 768] ~ N(0, 1); the seeds of the w1, w3, w2
    matvecs of the decode set's layer (workload 2, tensors 4, 5, 6)."""
    w1 = normal((LLAMA_HIDDEN, LLAMA_DIM), seed_of(2, layer, 4), W_STD, device)
    w3 = normal((LLAMA_HIDDEN, LLAMA_DIM), seed_of(2, layer, 5), W_STD, device)
    w2 = normal((LLAMA_DIM, LLAMA_HIDDEN), seed_of(2, layer, 6), W_STD, device)
    x = normal((n_tok, LLAMA_DIM), seed_of(2, layer, 7), 1.0, device)
    return dict(w1=w1, w3=w3, w2=w2, x=x)


def moe_layer_tensors(c: int, layer: int, shape: MoeShape, n_tok: int, x_std: float,
                      device="cpu"):
    """fp32 tensors of one MoE (or dense, n_exp == 1) FFN layer.

    Returns dict: up_gate [n_exp, 2*n_ff, n_embd], down [n_exp, n_embd, n_ff],
    x [n_tok, n_embd], ids [n_tok, n_used] int32 (None when dense),
    p [n_tok, n_used] fp32 (None when dense)."""
    ug = normal((shape.n_exp, 2 * shape.n_ff, shape.n_embd), seed_of(c, layer, 0), W_STD, device)
    dn = normal((shape.n_exp, shape.n_embd, shape.n_ff), seed_of(c, layer, 1), W_STD, device)
    x = normal((n_tok, shape.n_embd), seed_of(c, layer, 2), x_std, device)
    if shape.n_exp > 1:
        ids = routing_ids(n_tok, shape.n_exp, shape.n_used, seed_of(c, layer, 3))
        p = routing_weights(n_tok, shape.n_used, seed_of(c, layer, 4))
    else:
        ids, p = None, None
    return dict(up_gate=ug, down=dn, x=x, ids=ids, p=p)
