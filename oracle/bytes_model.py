"""Storage arithmetic.

kv_cache_bytes: [ru "Сколько памяти занимает KV-кэш"] gives the dense cache size as
2 x num_layers x num_kv_heads x d_head x seq_len x dtype_bytes.

cell_bytes: bytes a compressed cell stores. The pages give no formula; reading (written out from
what a cell holds [v4 §3]): token basis U_T [T, r_T], feature basis U_d [d_h, r_d] and core
G [L_g, n_kv, r_T, r_d] in the factor dtype, plus — when b > 0 — one packed b-bit code per
residual element and one 4-byte (fp16 scale, fp16 zero) pair per quantised row of d_h values.
The 4 bytes per quantised vector match the int8 baseline's ratio 2T/(T+4) [v4 App. E].

Pinned by: 327,680 B/token for Llama-3.1-70B (40 GiB at 128K) and 2,621,440 B/token without GQA
[ru "Сколько памяти занимает KV-кэш"]; 268.4 MB for Mistral-7B at ctx 2048 [nl Resultaten,
Efficiëntie]; the int8 ratio 2d/(d+4) for a residual-only 8-bit cell [v4 App. E].
"""


def kv_cache_bytes(n_layers: int, n_kv: int, d_head: int, seq_len: int, dtype_bytes: int) -> int:
    return 2 * n_layers * n_kv * d_head * seq_len * dtype_bytes


def raw_sequence_bytes(w) -> int:
    """Dense K+V bytes of one sequence of workload w in its I/O dtype."""
    return kv_cache_bytes(w.n_layers, w.n_kv, w.d_h, w.T, w.io_bytes)


def cell_bytes(T: int, d_h: int, L_g: int, n_kv: int, s_f: int, r_T: int, r_d: int, b: int) -> int:
    factors = s_f * (T * r_T + d_h * r_d + L_g * n_kv * r_T * r_d)
    resid = L_g * n_kv * T * (d_h * b // 8 + 4) if b > 0 else 0
    return factors + resid
