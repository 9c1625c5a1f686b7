"""The five synthetic workloads: shapes, dtypes, spectra and the rank/bit or budget setting.

Shapes follow the head geometry of the models the JoLT pages evaluate (Llama-3.1-8B: 32 query
heads, 8 KV heads, d_h=128; Llama-3.1-70B: 80 layers, 64 query heads, 8 KV heads) at the context
lengths of the long-context experiments. The data is a planted low-rank signal plus Gaussian noise
(X[l,h] = P_l diag(s_l) C_{l,h} Q_l^T + 0.05 N(0,1)), which stands in for real prefill caches.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_layers: int
    layers_per_group: int
    n_kv: int
    n_q: int
    T: int
    d_h: int
    io_dtype: str              # "f32" or "bf16": dtype of K, V, q and the attention output
    factor_dtype: str          # dtype the Tucker factors are stored in
    rank: int                  # planted rank R of every (layer, head) slice
    k_decay: Tuple[float, float]   # spectrum decay s_i = d**i, d ~ U[lo, hi] per layer (lo == hi: fixed)
    v_decay: Tuple[float, float]
    keys_pre_rope: bool
    rope_theta: float = 500000.0
    fixed_choice: Optional[Tuple[int, int, int]] = None   # (r_T, r_d, b) for every cell, else allocator
    budget_ratios: Tuple[float, ...] = ()
    seed: int = 0
    q_cap: int = 1024          # token-rank cap of the randomized token-mode SVD
    oversample: int = 128      # extra sketch columns beyond q_cap
    power_iters: int = 3
    noise: float = 0.05
    outlier_scale: float = 10.0
    tags: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def n_groups(self) -> int:
        return self.n_layers // self.layers_per_group

    @property
    def gq(self) -> int:
        return self.n_q // self.n_kv

    @property
    def n_cols(self) -> int:
        """Columns of the token-mode unfolding of one cell: L_g * n_kv * d_h."""
        return self.layers_per_group * self.n_kv * self.d_h

    @property
    def io_bytes(self) -> int:
        return 4 if self.io_dtype == "f32" else 2

    @property
    def factor_bytes(self) -> int:
        return 4 if self.factor_dtype == "f32" else 2

    @property
    def qcap_eff(self) -> int:
        return min(self.q_cap, self.n_cols, self.T)

    @property
    def sketch_cols(self) -> int:
        return min(self.qcap_eff + self.oversample, self.n_cols, self.T)

    def group_first_layers(self):
        return [g * self.layers_per_group for g in range(self.n_groups + 1)]


WORKLOADS = {
    # Toy single group: 1 layer, 2 KV heads, 4 q-heads per KV head, fp32, fixed ranks.
    "toy": Workload(
        name="toy", batch=1, n_layers=1, layers_per_group=1, n_kv=2, n_q=8, T=256, d_h=64,
        io_dtype="f32", factor_dtype="f32", rank=16, k_decay=(0.8, 0.8), v_decay=(0.95, 0.95),
        keys_pre_rope=False, fixed_choice=(32, 32, 4), seed=0),
    # Llama-3.1-8B-shaped single layer, T=4096, full token rank r_T = n = 1024.
    "llama8b_layer": Workload(
        name="llama8b_layer", batch=1, n_layers=1, layers_per_group=1, n_kv=8, n_q=32, T=4096,
        d_h=128, io_dtype="bf16", factor_dtype="bf16", rank=128, k_decay=(0.97, 0.97),
        v_decay=(0.97, 0.97), keys_pre_rope=False, fixed_choice=(1024, 96, 4), seed=1),
    # 8B-shaped, 32 layers in groups of 4, T=32768, allocator at a 3x budget.
    "llama8b_32k": Workload(
        name="llama8b_32k", batch=1, n_layers=32, layers_per_group=4, n_kv=8, n_q=32, T=32768,
        d_h=128, io_dtype="bf16", factor_dtype="bf16", rank=128, k_decay=(0.95, 0.99),
        v_decay=(0.95, 0.99), keys_pre_rope=False, budget_ratios=(3.0,), seed=2),
    # 8B-shaped, T=65536, batch 4, pre-RoPE keys, budgets 3x and 5x.
    "llama8b_64k_b4": Workload(
        name="llama8b_64k_b4", batch=4, n_layers=32, layers_per_group=4, n_kv=8, n_q=32, T=65536,
        d_h=128, io_dtype="bf16", factor_dtype="bf16", rank=128, k_decay=(0.95, 0.99),
        v_decay=(0.95, 0.99), keys_pre_rope=True, budget_ratios=(3.0, 5.0), seed=3),
    # Llama-3.1-70B-shaped, 80 layers, T=131072 (40 GiB raw), pre-RoPE keys, flat values, 3x.
    "llama70b_128k": Workload(
        name="llama70b_128k", batch=1, n_layers=80, layers_per_group=4, n_kv=8, n_q=64, T=131072,
        d_h=128, io_dtype="bf16", factor_dtype="bf16", rank=128, k_decay=(0.95, 0.99),
        v_decay=(0.99, 0.99), keys_pre_rope=True, budget_ratios=(3.0,), seed=4),
}

ORDER = ["toy", "llama8b_layer", "llama8b_32k", "llama8b_64k_b4", "llama70b_128k"]


def get_workload(name_or_index, **overrides) -> Workload:
    if isinstance(name_or_index, int):
        name_or_index = ORDER[name_or_index]
    w = WORKLOADS[name_or_index]
    if overrides:
        d = {k: getattr(w, k) for k in w.__dataclass_fields__}
        d.update(overrides)
        w = Workload(**d)
    return w
