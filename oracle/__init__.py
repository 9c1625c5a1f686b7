"""CPU oracle for the JoLT KV-cache codec — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 NumPy restatement of what the codec computes, written from the JoLT pages:

* "A JoLT for the KV cache: Near-Lossless KV Cache Compression via Joint Rank-bit Allocation"
  (paperlayer.ai summary of arXiv:2607.12550v4), cited as [v4 §n];
* "Technische Samenvatting: Een JOLT voor de KV Cache" (gist.science/nl), cited as [nl Methodologie];
* "JoLT: совместное распределение ранга и бит в KV-кэше" (sarnas.ru blog), cited as [ru <section>].

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg may import this
package. It shares no code with the CUDA library and imports nothing from it.

Parity status per function is stated in each module's header; every function here is pinned by
a `-m "not gpu"` test to something other than itself (closed forms, invariants, brute force, or
values the pages print), except where a header says "parity unpinned".
"""
from .rng import splitmix64, rotation_signs  # noqa: F401
from .rotation import hadamard, rotation_matrix  # noqa: F401
from .bytes_model import kv_cache_bytes, cell_bytes, raw_sequence_bytes  # noqa: F401
from .hosvd import token_unfolding, st_hosvd, spectra_tails, reconstruct  # noqa: F401
from .quant import quantize_rows, dequantize_rows, pack_codes, unpack_codes, phi_table  # noqa: F401
from .alloc import build_options, allocate, brute_force_allocate, allocate_kv_split, allocate_uniform, allocate_coord  # noqa: F401
from .codec import compress_cell, decompress_cell, decompress_slice, decode_attention, rope  # noqa: F401
from .grouping import layer_token_basis, subspace_alignment, layer_alignment, group_layers, uniform_group  # noqa: F401
