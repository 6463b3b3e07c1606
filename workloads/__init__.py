"""Seeded synthetic inputs for the masked INT8 linear, shared by the tests, the bench and
the oracle-side checks.

This module holds workload *shapes* and *random draws* only: no step of the method's
arithmetic (no Hadamard, no quantizer, no mask, no GEMM) lives here, so the oracle and the
CUDA path can both be fed from it without sharing any of the computation under test.

The five workloads mirror the model shapes the pages evaluate on:
  * "single"    - one linear, 256 tokens, 1152 -> 1152, 4 steps with bits {8,6,5,4}.
  * "pixart"    - PixArt-Sigma-shaped DiT (TASQ, "Resultados Experimentais": PixArt-Sigma 0.6B),
                  28 blocks x {qkv, proj, fc1, fc2}, batch 2 x 4096 tokens, 20 steps.
  * "sana"      - SANA-1.6B-shaped stack (same TASQ section), hidden 2240, 20 blocks, 20 steps,
                  Hadamard block 128.
  * "sdxl"      - SDXL-Turbo-shaped UNet transformer linears (same TASQ section), batch 4 x 1024
                  tokens, 4 steps, heavy-tailed Student-t channels.
  * "cogvideox" - CogVideoX-5B-shaped video DiT (6Bit-Diffusion, "Resultados Experimentais"),
                  17776 tokens, 42 blocks, 50 steps, bits in {8, 4} by a relative-L1 rule.

The pages publish no datasets we could use here (MJHQ-30K, sDCI, ImageNet, LSUN, COCO are
quality benchmarks that need trained weights); these synthetic tensors stand in for the
activations and weights those runs would feed the linear layers.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

import numpy as np

DATA_SEED = 0
SCHEDULE_SEED = 1

# tags that separate the random streams of different tensors
_TAG_ACT = 11
_TAG_OUTLIER_COLS = 12
_TAG_W = 21
_TAG_SW = 22
_TAG_SCHED = 31


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    tokens: int                              # M = batch x sequence
    block_layers: Tuple[Tuple[str, int, int], ...]   # (name, K in-features, N out-features)
    blocks: int
    steps: int
    hadamard_n: int
    schedule_kind: str                       # "fixed", "biased_high", "uniform", "relative_l1"
    fixed_bits: Tuple[int, ...] = ()         # per step, for schedule_kind == "fixed"
    outlier_kind: str = "scale50"            # "scale50" or "student_t3"
    outlier_frac: float = 0.005
    # groups of block-layer indices that read the same input (one prologue feeds their GEMMs)
    shared_input: Tuple[Tuple[int, ...], ...] = ()
    # relative_l1 schedules: the width of the stable blocks (0 = the NVFP4 step)
    stable_bits: int = 4
    # the on-device predictor picks every block's format at every step (INT8 8 bits or NVFP4)
    dmpq_online: bool = False

    def forward_plan(self) -> List[Tuple[int, ...]]:
        """The block's linears in order, as tuples of block-layer indices sharing one input."""
        lead = {g[0]: g for g in self.shared_input}
        members = {j for g in self.shared_input for j in g}
        plan = []
        for j in range(len(self.block_layers)):
            if j in lead:
                plan.append(tuple(lead[j]))
            elif j not in members:
                plan.append((j,))
        return plan

    @property
    def num_layers(self) -> int:
        return self.blocks * len(self.block_layers)

    def layer_shape(self, layer: int) -> Tuple[str, int, int]:
        return self.block_layers[layer % len(self.block_layers)]

    def kp(self, K: int) -> int:
        """K rounded up to whole Hadamard blocks (zero padding of the activations)."""
        n = self.hadamard_n
        return -(-K // n) * n

    def gemm_ops_per_step(self) -> int:
        """2*M*N*K integer ops per step, counted at the unpadded K."""
        return 2 * self.tokens * self.blocks * sum(K * N for _, K, N in self.block_layers)

    def prologue_bytes_per_step(self) -> int:
        """Algorithmic prologue bytes per step: 2K read + Kp codes + 4 scale per token and input
        (linears sharing an input quantize it once)."""
        return self.tokens * self.blocks * sum(
            2 * K + self.kp(K) + 4 for K in (self.block_layers[g[0]][1] for g in self.forward_plan()))


WORKLOADS = {
    "single": Workload(
        name="single", tokens=256, block_layers=(("linear", 1152, 1152),), blocks=1, steps=4,
        hadamard_n=64, schedule_kind="fixed", fixed_bits=(8, 6, 5, 4)),
    "pixart": Workload(
        name="pixart", tokens=2 * 4096,
        block_layers=(("qkv", 1152, 3456), ("proj", 1152, 1152), ("fc1", 1152, 4608), ("fc2", 4608, 1152)),
        blocks=28, steps=20, hadamard_n=64, schedule_kind="biased_high"),
    "sana": Workload(
        name="sana", tokens=2 * 1024,
        block_layers=(("qkv", 2240, 6720), ("proj", 2240, 2240), ("fc1", 2240, 5600), ("fc2", 5600, 2240)),
        blocks=20, steps=20, hadamard_n=128, schedule_kind="uniform"),
    "sdxl": Workload(
        name="sdxl", tokens=4 * 1024,
        block_layers=(("q", 1280, 1280), ("k", 1280, 1280), ("v", 1280, 1280), ("out", 1280, 1280),
                      ("ff_geglu", 1280, 10240), ("ff_out", 5120, 1280)),
        blocks=1, steps=4, hadamard_n=64, schedule_kind="fixed", fixed_bits=(8, 6, 5, 4),
        outlier_kind="student_t3", outlier_frac=0.01, shared_input=((0, 1, 2),)),
    "cogvideox": Workload(
        name="cogvideox", tokens=13 * 30 * 45 + 226,
        block_layers=(("qkv", 3072, 9216), ("proj", 3072, 3072), ("fc1", 3072, 12288), ("fc2", 12288, 3072)),
        blocks=42, steps=50, hadamard_n=64, schedule_kind="relative_l1"),
    # 6Bit-Diffusion's own split on the same shapes: unstable blocks in INT8, stable ones in NVFP4
    "cogvideox_nvfp4": Workload(
        name="cogvideox_nvfp4", tokens=13 * 30 * 45 + 226,
        block_layers=(("qkv", 3072, 9216), ("proj", 3072, 3072), ("fc1", 3072, 12288), ("fc2", 12288, 3072)),
        blocks=42, steps=50, hadamard_n=64, schedule_kind="relative_l1", stable_bits=0),
    # the same split decided on the device each step by the DMPQ predictor (the whole
    # 6Bit-Diffusion loop): block b's relative L1 change is taken between its input and the next
    # block's input, the threshold is the median over the blocks of the first step
    "cogvideox_dmpq": Workload(
        name="cogvideox_dmpq", tokens=13 * 30 * 45 + 226,
        block_layers=(("qkv", 3072, 9216), ("proj", 3072, 3072), ("fc1", 3072, 12288), ("fc2", 12288, 3072)),
        blocks=42, steps=50, hadamard_n=64, schedule_kind="relative_l1", stable_bits=0, dmpq_online=True),
}

# order of the INT8 workloads as the task lists them (cogvideox_nvfp4 is the NVFP4 variant)
WORKLOAD_ORDER = ("single", "pixart", "sana", "sdxl", "cogvideox")


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(list(key))


def outlier_columns(wl: Workload, K: int, layer: int, seed: int = DATA_SEED) -> np.ndarray:
    """Seeded set of input channels that carry outliers (0.5 % or 1 % of K)."""
    count = int(round(wl.outlier_frac * K))
    r = _rng(seed, _TAG_OUTLIER_COLS, layer, K)
    return np.sort(r.choice(K, size=count, replace=False))


def activations(wl: Workload, layer: int, M: int | None = None, seed: int = DATA_SEED) -> np.ndarray:
    """FP16 activations [M, K] for `layer`: N(0,1) with outlier channels.

    scale50    : the outlier channels are multiplied by 50.
    student_t3 : the outlier channels are replaced by Student-t draws with nu = 3.
    Drawn in float32 and cast to float16 with round-to-nearest-even.
    """
    _, K, _ = wl.layer_shape(layer)
    M = wl.tokens if M is None else M
    r = _rng(seed, _TAG_ACT, layer)
    x = r.standard_normal((M, K), dtype=np.float32)
    cols = outlier_columns(wl, K, layer, seed)
    if wl.outlier_kind == "scale50":
        x[:, cols] *= np.float32(50.0)
    elif wl.outlier_kind == "student_t3":
        x[:, cols] = r.standard_t(3.0, size=(M, cols.size)).astype(np.float32)
    else:
        raise ValueError(wl.outlier_kind)
    return x.astype(np.float16)


def weights(wl: Workload, layer: int, seed: int = DATA_SEED) -> Tuple[np.ndarray, np.ndarray]:
    """INT8 weight codes [N, Kp] uniform in [-127, 127] and FP32 scales [N] ~ U(0.001, 0.01).

    The codes fill all Kp columns: the stored buffer lives in the Hadamard-rotated basis, where
    the zero-padded tail of the activations mixes with every column.
    """
    _, K, N = wl.layer_shape(layer)
    Kp = wl.kp(K)
    w = _rng(seed, _TAG_W, layer).integers(-127, 128, size=(N, Kp), dtype=np.int8)
    s_w = _rng(seed, _TAG_SW, layer).uniform(0.001, 0.01, size=N).astype(np.float32)
    return w, s_w


def schedule(wl: Workload, seed: int = SCHEDULE_SEED) -> np.ndarray:
    """Effective weight bits per (layer, step), uint8 [num_layers, steps], each in [0, 8]
    (0: the NVFP4 step).

    fixed       : the same bits for every layer at step t (single, sdxl: 8, 6, 5, 4).
    biased_high : clip(round(8 - 4 t / (T - 1) + N(0, 0.75)), 4, 8)  (pixart).
    uniform     : i.i.d. uniform over {4, ..., 8}, mean 6 (sana).
    relative_l1 : per (block, step) a synthetic relative-L1 block change Gamma ~ LogNormal(-3, 0.5);
                  Gamma above the median of all Gamma -> 8 bits, else stable_bits (4, or 0 for
                  NVFP4); step 0 has no previous step to measure and runs at 8; the linears of a
                  block share its bits (cogvideox, cogvideox_nvfp4).
    """
    L, T = wl.num_layers, wl.steps
    per_block = len(wl.block_layers)
    r = _rng(seed, _TAG_SCHED)
    if wl.schedule_kind == "fixed":
        assert len(wl.fixed_bits) == T
        bits = np.tile(np.asarray(wl.fixed_bits, dtype=np.int64), (L, 1))
    elif wl.schedule_kind == "biased_high":
        t = np.arange(T, dtype=np.float64)
        base = 8.0 - 4.0 * t / max(T - 1, 1)
        bits = np.clip(np.rint(base[None, :] + r.normal(0.0, 0.75, size=(L, T))), 4, 8).astype(np.int64)
    elif wl.schedule_kind == "uniform":
        bits = r.integers(4, 9, size=(L, T))
    elif wl.schedule_kind == "relative_l1":
        gamma = r.lognormal(mean=-3.0, sigma=0.5, size=(wl.blocks, T))
        thr = np.median(gamma)
        block_bits = np.where(gamma > thr, 8, wl.stable_bits)
        block_bits[:, 0] = 8
        bits = np.repeat(block_bits, per_block, axis=0)
    else:
        raise ValueError(wl.schedule_kind)
    return bits.astype(np.uint8)


def sample_rows(M: int, count: int = 128, seed: int = DATA_SEED, tile: int = 256) -> np.ndarray:
    """Seeded sample of token rows for full-size parity: `count` random rows plus every row of
    the last (possibly ragged) token tile."""
    r = _rng(seed, 41, M)
    pick = r.choice(M, size=min(count, M), replace=False)
    last = np.arange((M - 1) // tile * tile, M)
    return np.unique(np.concatenate([pick, last]))


# ---------------------------------------------------------------------------------------------
# device-side draws for the bench (timing data only; same recipe, torch's seeded generator)
# ---------------------------------------------------------------------------------------------
def activations_torch(wl: Workload, layer: int, device, seed: int = DATA_SEED, M: int | None = None):
    """Same recipe as `activations`, drawn on the device with torch's seeded generator.

    Used only where the values are not checked (bench timing buffers), because generating tens
    of GB on the host would dominate the run."""
    import torch
    _, K, _ = wl.layer_shape(layer)
    M = wl.tokens if M is None else M
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(layer) * 7919 + 17)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    cols = torch.from_numpy(outlier_columns(wl, K, layer, seed)).to(device)
    if wl.outlier_kind == "scale50":
        x[:, cols] *= 50.0
    else:
        # Student-t(3) = N / sqrt(chi2_3 / 3), chi2_3 as a sum of three squared normals
        z = torch.randn((M, cols.numel()), generator=g, device=device)
        c = torch.randn((3, M, cols.numel()), generator=g, device=device).square().sum(0)
        x[:, cols] = z / torch.sqrt(c / 3.0)
    return x.to(torch.float16)


def weights_torch(wl: Workload, layer: int, device, seed: int = DATA_SEED):
    import torch
    _, K, N = wl.layer_shape(layer)
    Kp = wl.kp(K)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_033 + int(layer) * 104729 + 23)
    w = torch.randint(-127, 128, (N, Kp), generator=g, device=device, dtype=torch.int8)
    s_w = torch.empty(N, device=device, dtype=torch.float32).uniform_(0.001, 0.01, generator=g)
    return w, s_w


def describe(wl: Workload) -> dict:
    return {
        "workload": wl.name, "tokens": wl.tokens, "blocks": wl.blocks, "steps": wl.steps,
        "hadamard_n": wl.hadamard_n,
        "layers_per_block": [f"{n}:{K}->{N}" for n, K, N in wl.block_layers],
    }
