"""The workloads: weight sets shaped like the models the pages run.

The pages' experiments use a Qwen3-8B dense model (verl PR #4415, "Experiments
and Outcomes") and dense plus MoE models (FP8-RL abstract).  The quantizer
sees every linear weight and every fused-MoE expert weight of the rollout
model ("vllm_fp8_utils.py" docs, sections 2 and 3: is_fp8_weight and
quant_weights).  No checkpoint is available, so values are synthetic with the
statistics below; shapes are those of the named architectures.

  small       one bf16 256x384 matrix (2x3 blocks of 128x128) with an all-zero
              block, a block whose absmax is exactly 448 and a block scaled by
              1e-6.
  qwen3_8b    per layer q,k,v,o,gate,up,down (k, v: 8 KV heads x 128); values
              N(0, 0.02) x per-row lognormal(0, 0.5), 0.1% outliers
              +-U(0.5, 4); layer seeds 1 (one-layer case) or 100 + layer.
  moe_30b_a3b per layer q 4096x2048, k,v 512x2048, o 2048x4096, w13
              [128, 1536, 2048], w2 [128, 2048, 768]; N(0, 0.02) x per-expert
              lognormal(0, 0.7) (attention weights: factor 1); seed 2.
  edge        ragged bf16 and fp32 matrices with Student-t(3) x 0.02 values;
              16384x4096 bf16 N(0,1) x per-row lognormal(0,1) with blocks
              [1,128] and [64,64]; row-padded (ld = N + 64) variants; seed 3.
"""
from __future__ import annotations

import numpy as np

from . import DIST_STUDENT_T3, TensorSpec, f32_to_bf16_bits, fill_into

QWEN3_8B_LAYER = [  # (name, M = out_features, N = in_features)
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 12288, 4096),
    ("up_proj", 12288, 4096),
    ("down_proj", 4096, 12288),
]
QWEN3_8B_LAYERS = 36

MOE_LAYERS = 48


def small() -> list[TensorSpec]:
    """256x384 bf16, 2x3 blocks of 128x128, with three directed blocks."""
    return [TensorSpec("small", 256, 384, seed=0, tensor_id=0, sigma=0.02,
                       meta={"recipe": "small"})]


def _small_values(spec: TensorSpec) -> np.ndarray:
    base = TensorSpec(spec.name, spec.M, spec.N, dtype="f32", seed=spec.seed,
                      tensor_id=spec.tensor_id, sigma=spec.sigma)
    x = np.empty((spec.M, spec.N), dtype=np.float32)
    fill_into(base, x.ctypes.data)
    x[0:128, 128:256] = 0.0                                   # block (0,1): all +0
    blk = x[128:256, 256:384].astype(np.float64) * 1e-6       # block (1,2): x 1e-6
    x[128:256, 256:384] = blk.astype(np.float32)
    b10 = x[128:256, 0:128].astype(np.float64)                # block (1,0): absmax 448
    flat = int(np.argmax(np.abs(b10)))
    sign = 1.0 if b10.flat[flat] >= 0 else -1.0
    x[128:256, 0:128] = (b10 * (448.0 / np.abs(b10).max())).astype(np.float32)
    h = f32_to_bf16_bits(x)
    r, c = divmod(flat, 128)
    h[128 + r, c] = f32_to_bf16_bits(np.array([448.0 * sign], dtype=np.float32))[0]
    return h.reshape(-1)


def qwen3_8b_layer(layer: int = 0, seed: int | None = None) -> list[TensorSpec]:
    """One Qwen3-8B-shaped decoder layer's seven linear weights (bf16)."""
    seed = 1 if seed is None else seed
    return [TensorSpec(f"layers.{layer}.{name}", M, N, seed=seed, tensor_id=i,
                       sigma=0.02, row_lognormal_sigma=0.5, outlier_p=1e-3,
                       outlier_lo=0.5, outlier_hi=4.0, meta={"layer": layer})
            for i, (name, M, N) in enumerate(QWEN3_8B_LAYER)]


def qwen3_8b_model(layers: int = QWEN3_8B_LAYERS) -> list[TensorSpec]:
    """All linear weights of a Qwen3-8B-shaped model, layer seeds 100 + layer."""
    out: list[TensorSpec] = []
    for layer in range(layers):
        out += qwen3_8b_layer(layer, seed=100 + layer)
    return out


def moe_layer(layer: int = 0) -> list[TensorSpec]:
    """One Qwen3-30B-A3B-style MoE layer; experts are batch entries."""
    seed = 2
    tid = layer * 16
    att = dict(seed=seed, sigma=0.02, meta={"layer": layer})
    return [
        TensorSpec(f"layers.{layer}.q_proj", 4096, 2048, tensor_id=tid + 0, **att),
        TensorSpec(f"layers.{layer}.k_proj", 512, 2048, tensor_id=tid + 1, **att),
        TensorSpec(f"layers.{layer}.v_proj", 512, 2048, tensor_id=tid + 2, **att),
        TensorSpec(f"layers.{layer}.o_proj", 2048, 4096, tensor_id=tid + 3, **att),
        TensorSpec(f"layers.{layer}.experts.w13_weight", 1536, 2048, batch=128,
                   tensor_id=tid + 4, batch_lognormal_sigma=0.7, **att),
        TensorSpec(f"layers.{layer}.experts.w2_weight", 2048, 768, batch=128,
                   tensor_id=tid + 5, batch_lognormal_sigma=0.7, **att),
    ]


def edge() -> list[TensorSpec]:
    """Ragged shapes in bf16 and fp32, small-block cases and row-padded inputs."""
    out: list[TensorSpec] = []
    tid = 0
    for dtype in ("bf16", "f32"):
        for (M, N) in ((4000, 4100), (130, 129), (1, 128), (12345, 4096)):
            out.append(TensorSpec(f"edge.{dtype}.{M}x{N}", M, N, dtype=dtype, seed=3,
                                  tensor_id=tid, dist=DIST_STUDENT_T3, sigma=0.02))
            tid += 1
    for blk in ((1, 128), (64, 64)):
        out.append(TensorSpec(f"edge.bf16.16384x4096.b{blk[0]}x{blk[1]}", 16384, 4096,
                              block=blk, seed=3, tensor_id=100, sigma=1.0,
                              row_lognormal_sigma=1.0))
    for dtype in ("bf16", "f32"):   # ld = N + 64: padding columns hold a large poison
        out.append(TensorSpec(f"edge.{dtype}.4000x4100.ld4164", 4000, 4100, ld=4164,
                              dtype=dtype, seed=3, tensor_id=200 + (dtype == "f32"),
                              dist=DIST_STUDENT_T3, sigma=0.02))
    return out


def qkv_activations(tokens: int = 16384) -> list[TensorSpec]:
    """Q, K, V activations of one Qwen3-8B-shaped attention layer for a batch of
    `tokens` tokens (Q: 32 heads x 128, K and V: 8 KV heads x 128), bf16,
    N(0,1) x per-token lognormal(0,1): the inputs of the per-step KV-cache
    scale recalibration."""
    return [TensorSpec(f"act.{name}", tokens, width, seed=4, tensor_id=i, sigma=1.0,
                       row_lognormal_sigma=1.0)
            for i, (name, width) in enumerate((("q", 4096), ("k", 1024), ("v", 1024)))]


def materialize(spec: TensorSpec, nthreads: int | None = None) -> np.ndarray:
    """Host array for ``spec`` (flat, numel_storage elements)."""
    if spec.meta.get("recipe") == "small":
        return _small_values(spec)
    a = np.empty(spec.numel_storage, dtype=spec.np_dtype)
    fill_into(spec, a.ctypes.data, nthreads)
    return a


def materialize_into(spec: TensorSpec, ptr: int, nthreads: int | None = None) -> None:
    """Write ``spec`` into host memory at ``ptr`` (e.g. a pinned torch tensor)."""
    if spec.meta.get("recipe") == "small":
        a = _small_values(spec)
        import ctypes
        ctypes.memmove(ptr, a.ctypes.data, a.nbytes)
        return
    fill_into(spec, ptr, nthreads)
