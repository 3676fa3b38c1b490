"""The benchmark workloads and their algorithmic work (visible pairs, flops, bytes).

Shapes follow the pages: 16 query heads over 4 key/value heads, head_dim 256
(system1-omni issue #27, "The closest planned or implemented model"); state lengths
15,231 / 30,468 / 60,926 tokens (kev PR #202, "Measurements"); a state followed by
8 question branches (system1-omni issue #27, item 3); 1,048,576-token packed
sequences (maxtext PR #4929, description).  Inputs are the seeded synthetic
tensors of ``inputs``; the documents and training data of the pages are not used.

Algorithmic work counts only visible (query, key) pairs: 4 * d * Hq flops per pair
(QK^T and PV, 2 d each), no exp / max work, no masked work inside partial tiles and
none of the L x L work the method avoids.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

HQ, HKV, D = 16, 4, 256


@dataclass
class Workload:
    name: str
    Lq: int
    Lk: int
    dtype: torch.dtype
    mask_kind: str = "causal"
    q_pos_offset: int = 0
    segments: list = field(default_factory=list)   # self-attention packing: segment lengths
    branches: tuple = ()                            # (n_branches, branch_len) after the state
    B: int = 1
    Hq: int = HQ
    Hkv: int = HKV
    d: int = D

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == torch.float32 else 2

    def visible_pairs(self) -> int:
        """Visible (query, key) pairs per head, in closed form."""
        if self.branches:
            nb, bl = self.branches
            return nb * bl * self.q_pos_offset + nb * bl * (bl + 1) // 2
        if self.segments:
            return sum(s * (s + 1) // 2 for s in self.segments)
        return self.Lq * self.q_pos_offset + self.Lq * (self.Lq + 1) // 2

    def flops(self) -> int:
        return 4 * self.d * self.Hq * self.visible_pairs() * self.B

    def io_bytes(self) -> int:
        """Minimum HBM traffic: Q, K, V read once, out and LSE written once (+ ids)."""
        e = self.elem_bytes
        q = self.B * self.Hq * self.Lq * self.d * e
        kv = 2 * self.B * self.Hkv * self.Lk * self.d * e
        lse = self.B * self.Hq * self.Lq * 4
        ids = (self.Lq + self.Lk) * 4 if (self.segments or self.branches) else 0
        return 2 * q + kv + lse + ids


def causal(L, dtype, name=None, B=1):
    return Workload(name or f"causal_L{L}_{'f32' if dtype == torch.float32 else 'bf16'}", L, L, dtype, B=B)


def branches_after_state(state_len=30_468, n_branches=8, branch_len=256, dtype=torch.float32):
    Lq = n_branches * branch_len
    return Workload(f"branches_{n_branches}x{branch_len}_after_{state_len}", Lq, state_len + Lq, dtype,
                    mask_kind="prefix_branch", q_pos_offset=state_len, branches=(n_branches, branch_len))


def segmented(L, lengths, dtype=torch.bfloat16, name=None):
    assert sum(lengths) == L
    return Workload(name or f"segmented_L{L}", L, L, dtype, segments=list(lengths))


# The five configurations (the fourth in both dtypes; the fifth with seeded
# segment lengths and with one constant-id segment).
def configs():
    from .inputs import segment_lengths

    L5 = 1_048_576
    cfg = {
        "causal_512_f32": causal(512, torch.float32),
        "causal_15231_f32": causal(15_231, torch.float32),
        "state_30468_f32": causal(30_468, torch.float32),
        "branches_8x256_after_30468_f32": branches_after_state(),
        "branches_8x256_after_30468_bf16": branches_after_state(dtype=torch.bfloat16),
        "causal_60926_f32": causal(60_926, torch.float32),
        "causal_60926_bf16": causal(60_926, torch.bfloat16),
        "segmented_1M_bf16": segmented(L5, segment_lengths(L5)),
        "constant_ids_1M_bf16": segmented(L5, [L5]),
        "causal_1M_bf16": causal(L5, torch.bfloat16),
    }
    for name, w in cfg.items():
        w.name = name
    return cfg


def by_name(name):
    """A configuration above, or ``causal_<L>_<f32|bf16>`` for any length (profiling sizes)."""
    cfg = configs()
    if name in cfg:
        return cfg[name]
    parts = name.split("_")
    if len(parts) == 3 and parts[0] == "causal" and parts[1].isdigit() and parts[2] in ("f32", "bf16"):
        w = causal(int(parts[1]), torch.float32 if parts[2] == "f32" else torch.bfloat16)
        w.name = name
        return w
    raise KeyError(f"unknown workload {name}; choose from {sorted(cfg)} or causal_<L>_<f32|bf16>")
