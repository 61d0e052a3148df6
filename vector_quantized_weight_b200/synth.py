"""Seeded synthetic inputs for the VQ decode linear.

This module only draws random tensors in the canonical layouts; it holds none
of the method's arithmetic, so both the double-precision oracle and the CUDA
path consume exactly the same bytes.

Canonical layouts (shared by the oracle and the C ABI):
  wc     fp16  [G][256][d]     weight codebook WC, G = N / codebook_rows or 1
  wi     uint8 [N][K/d]        weight-index matrix WI, row-major
  x      fp16  [B][K]          decode-step activations
  signs  uint8 [N][K/8]        1-bit residual signs, LSB-first along k
                               (bit i of byte m is k = 8m + i; 1 -> +1, 0 -> -1)
  alpha  fp16  [N][K/128]      residual scale per 128-input group
  hsign  int8  [K]             +-1 diagonal of the randomized Hadamard

Distributions follow the decode workloads of the EVA summary (section 4:
LLaMA-family linears) and of the 3-bit SRAM-lookup article (Gemma-2-9B,
d=4 / 256-centroid product quantization, 1-bit sign residual, fp16 alpha per
128-group): WC ~ N(0, 0.02^2), WI ~ U{0..255}, x ~ N(0, 1),
|alpha| ~ U(0.001, 0.01), uniform sign bits, uniform +-1 Hadamard signs.
No real weights or datasets are used; the shapes alone stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BASE_SEED = 20260526


@dataclass(frozen=True)
class LayerShape:
    """One linear layer: N outputs, K inputs, plus the quantization format."""
    name: str
    N: int
    K: int
    d: int = 4
    codebook_rows: int = 0      # 0: one shared codebook; 128: one per 128 output rows
    residual_group: int = 0     # 0: no sign residual; 128: signs + alpha per 128 inputs
    hadamard_block: int = 0     # 0: no rotation; else block size b of the rotation
    index_bits: int = 8         # 8: one index byte per sub-vector; 4: 16 centroids, two per byte

    @property
    def J(self) -> int:
        return self.K // self.d

    @property
    def G(self) -> int:
        return self.N // self.codebook_rows if self.codebook_rows else 1

    @property
    def ncent(self) -> int:
        return 1 << self.index_bits


@dataclass(frozen=True)
class Config:
    """A named workload: a list of layers and the batch sizes it is run at."""
    key: str
    title: str
    layers: tuple
    batches: tuple = (1,)
    index: int = 0              # seed offset: seed = BASE_SEED + 100*index + layer


def _llama7b_block():
    return (
        LayerShape("q_proj", 4096, 4096), LayerShape("k_proj", 4096, 4096),
        LayerShape("v_proj", 4096, 4096), LayerShape("o_proj", 4096, 4096),
        LayerShape("gate_proj", 11008, 4096), LayerShape("up_proj", 11008, 4096),
        LayerShape("down_proj", 4096, 11008),
    )


def _gemma_3bit():
    # 3584 = 7 * 512 and 14336 = 7 * 2048: the rotation block is the largest
    # power of two dividing K.
    return (
        LayerShape("gemma_3584x3584", 3584, 3584, residual_group=128, hadamard_block=512),
        LayerShape("gemma_14336x3584", 14336, 3584, residual_group=128, hadamard_block=512),
        LayerShape("gemma_3584x14336", 3584, 14336, residual_group=128, hadamard_block=2048),
    )


def _gemma_3bit_order_k():
    # The same layers with the rotation over the whole input dimension:
    # 3584 = 28 * 128 and 14336 = 28 * 512, H_K = H28 (x) H_(K/28).
    return (
        LayerShape("gemma_3584x3584_rotK", 3584, 3584, residual_group=128, hadamard_block=3584),
        LayerShape("gemma_14336x3584_rotK", 14336, 3584, residual_group=128, hadamard_block=3584),
        LayerShape("gemma_3584x14336_rotK", 3584, 14336, residual_group=128, hadamard_block=14336),
    )


def _llama70b():
    return (
        LayerShape("l70b_8192x8192", 8192, 8192, codebook_rows=128),
        LayerShape("l70b_28672x8192", 28672, 8192, codebook_rows=128),
        LayerShape("l70b_8192x28672", 8192, 28672, codebook_rows=128),
    )


CONFIGS = {
    "tiny": Config("tiny", "Tiny 2-bit VQ linear 256x512, batch 1",
                   (LayerShape("tiny_256x512", 256, 512),), (1,), 0),
    "llama7b_layer": Config("llama7b_layer", "Llama-2-7B-shaped 4096x4096 2-bit layer, batch 1",
                            (LayerShape("l7b_4096x4096", 4096, 4096),), (1,), 1),
    "llama7b_block": Config("llama7b_block", "All seven Llama-2-7B decoder-block linears, 2-bit",
                            _llama7b_block(), (1, 4, 16), 2),
    "gemma_3bit": Config("gemma_3bit", "Gemma-2-9B-shaped 3.125-bit linears (Hadamard + sign residual)",
                         _gemma_3bit(), (1,), 3),
    "llama70b": Config("llama70b", "Llama-2-70B-shaped 2-bit linears, one codebook per 128 rows",
                       _llama70b(), (1, 8, 32), 4),
    "llama7b_layer_4bit": Config("llama7b_layer_4bit", "Llama-2-7B-shaped 4096x4096 layer with 4-bit indices "
                                 "(16 centroids, 1 bit per weight), batch 1 and 4",
                                 (LayerShape("l7b_4096x4096_idx4", 4096, 4096, index_bits=4),), (1, 4), 6),
    "gemma_3bit_rotK": Config("gemma_3bit_rotK", "Gemma-2-9B-shaped 3.125-bit linears, order-K (Paley x "
                              "Sylvester) rotation", _gemma_3bit_order_k(), (1, 2), 5),
}


def layer_seed(config_index: int, layer_index: int) -> int:
    return BASE_SEED + 100 * config_index + layer_index


@dataclass
class LayerData:
    shape: LayerShape
    wc: np.ndarray
    wi: np.ndarray
    signs: np.ndarray | None
    alpha: np.ndarray | None
    hsign: np.ndarray | None
    seed: int = 0
    extra: dict = field(default_factory=dict)


def make_layer(shape: LayerShape, seed: int, *, alpha_signed: bool = False) -> LayerData:
    """Draw the weights of one layer. Order: WC, WI, signs, alpha, hsign."""
    rng = np.random.default_rng(seed)
    wc = rng.normal(0.0, 0.02, size=(shape.G, shape.ncent, shape.d)).astype(np.float16)
    wi = rng.integers(0, shape.ncent, size=(shape.N, shape.J), dtype=np.uint8)
    if shape.index_bits == 4:       # packed: sub-vector 2t in the low nibble of byte t
        wi = pack_nibbles(wi)
    signs = alpha = hsign = None
    if shape.residual_group:
        signs = rng.integers(0, 256, size=(shape.N, shape.K // 8), dtype=np.uint8)
        a = rng.uniform(0.001, 0.01, size=(shape.N, shape.K // shape.residual_group))
        if alpha_signed:
            a = a * (rng.integers(0, 2, size=a.shape) * 2 - 1)
        alpha = a.astype(np.float16)
    if shape.hadamard_block:
        hsign = (rng.integers(0, 2, size=shape.K) * 2 - 1).astype(np.int8)
    return LayerData(shape, wc, wi, signs, alpha, hsign, seed)


def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """[N][J] indices < 16 -> [N][J/2] bytes, even sub-vector in the low nibble."""
    idx = np.asarray(idx, dtype=np.uint8)
    return (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)


def make_x(K: int, B: int, seed: int) -> np.ndarray:
    """Activations x ~ N(0, 1) as fp16 [B][K], from their own stream."""
    rng = np.random.default_rng(seed + 7_000_000)
    return rng.normal(0.0, 1.0, size=(B, K)).astype(np.float16)


def adversarial_wi(N: int, J: int, pattern: str, seed: int = 0) -> np.ndarray:
    """Index matrices for the bit-exact repack round trip."""
    if pattern == "zeros":
        return np.zeros((N, J), np.uint8)
    if pattern == "ones":
        return np.full((N, J), 0xFF, np.uint8)
    if pattern == "a5":
        return np.full((N, J), 0xA5, np.uint8)
    if pattern == "ramp":
        return (np.arange(N * J, dtype=np.int64) % 256).astype(np.uint8).reshape(N, J)
    if pattern == "rowcol":
        o = np.arange(N)[:, None]
        j = np.arange(J)[None, :]
        return ((o * 7 + j * 13) % 256).astype(np.uint8)
    if pattern == "random":
        return np.random.default_rng(seed).integers(0, 256, size=(N, J), dtype=np.uint8)
    raise ValueError(pattern)


# ------------------------------------------------------- quantizer inputs

def make_dense_weight(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """A dense fp16 weight [N][K] ~ N(0, std^2) for the offline quantizer."""
    rng = np.random.default_rng(seed + 9_000_000)
    return rng.normal(0.0, std, size=(N, K)).astype(np.float16)


def make_hsign(K: int, seed: int) -> np.ndarray:
    """Rotation signs s [K] in {-1, +1} (int8)."""
    rng = np.random.default_rng(seed + 8_000_000)
    return rng.choice(np.array([-1, 1], np.int8), size=K)


def kmeans_init_index(vecs_per_cb: int, G: int, ncent: int, seed: int) -> np.ndarray:
    """Starting blocks of the K-means: for each of the G codebooks, ncent
    distinct block indices in [0, vecs_per_cb), drawn without replacement
    (int32 [G][ncent])."""
    rng = np.random.default_rng(seed + 7_500_000)
    return np.stack([rng.choice(vecs_per_cb, size=ncent, replace=False) for _ in range(G)]).astype(np.int32)
