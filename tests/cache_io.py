"""Test glue: lay the oracle's compressed cells out in the device cache layout, and run the
oracle's decode over whole workloads. Offsets come from the library's jolt_cache_layout; no
codec arithmetic lives here."""
import numpy as np
import torch

import oracle
from long_context_st_b200 import api

_FDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def cell_index(w, b, g, kv):
    return (b * (w.n_layers // w.layers_per_group) + g) * 2 + kv


def oracle_cells(w, K, V, choices, rot_seed, factor_dtype=None):
    """Compress every cell with the oracle. K, V: torch [B, L, n_kv, T, d_h] (any dtype)."""
    fdt = factor_dtype or w.factor_dtype
    G = w.n_layers // w.layers_per_group
    cells = []
    for b in range(K.shape[0]):
        for g in range(G):
            sl = slice(g * w.layers_per_group, (g + 1) * w.layers_per_group)
            for kv, X in ((0, K), (1, V)):
                c = choices[cell_index(w, b, g, kv)]
                Xc = X[b, sl].double().cpu().numpy()
                cells.append(oracle.compress_cell(Xc, c[0], c[1], c[2], rot_seed, fdt))
    return cells


def cells_to_device(shape, w, cells, choices, device="cuda", factor_dtype=None):
    """Write the oracle cells into one uint8 device buffer laid out by jolt_cache_layout."""
    fdt = _FDT[factor_dtype or w.factor_dtype]
    offs, total = api.cache_layout(shape, choices)
    buf = torch.zeros(total, dtype=torch.uint8)

    def put(off, t):
        raw = t.contiguous().view(torch.uint8).reshape(-1)
        buf[int(off):int(off) + raw.numel()] = raw

    for c, cell in enumerate(cells):
        rT, rd, b = choices[c]
        if rT:
            put(offs[c, 0], torch.from_numpy(np.ascontiguousarray(cell["U_T"])).to(fdt))
            put(offs[c, 1], torch.from_numpy(np.ascontiguousarray(cell["U_d"])).to(fdt))
            put(offs[c, 2], torch.from_numpy(np.ascontiguousarray(cell["G"])).to(fdt))
        if b:
            put(offs[c, 3], torch.from_numpy(np.ascontiguousarray(cell["codes"])))
            sz = np.stack([cell["scale"], cell["zero"]], axis=-1).astype(np.float16)
            put(offs[c, 4], torch.from_numpy(np.ascontiguousarray(sz)))
    return buf.to(device)


def parts_to_cells(w, parts_list, choices):
    """Random stored parts (synth.make_random_cache_parts) -> oracle cell dicts."""
    cells = []
    for parts, (rT, rd, b) in zip(parts_list, choices):
        d = w.d_h
        c = {"r_T": rT, "r_d": rd, "b": b,
             "shape": (w.layers_per_group, w.n_kv, w.T, d),
             "U_T": parts["U_T"].double().numpy(), "U_d": parts["U_d"].double().numpy(),
             "G": parts["G"].double().numpy()}
        if b:
            c["codes"] = parts["codes"].numpy()
            c["scale"] = parts["sz"][..., 0].numpy()
            c["zero"] = parts["sz"][..., 1].numpy()
        cells.append(c)
    return cells


def oracle_decode(w, cells, q, rot_seed, inv_freq=None, layers=None, heads=None, pos_offset=0,
                  attn_scale=None):
    """Oracle decode for every (b, layer, q-head) (or a subset). q: [B, L, n_q, d_h].
    Returns dict (b, layer) -> (out [n_q, d_h] or rows of `heads`, lse)."""
    G = w.n_layers // w.layers_per_group
    scale = attn_scale or 1.0 / np.sqrt(w.d_h)
    layers = range(w.n_layers) if layers is None else layers
    res = {}
    qn = q.double().cpu().numpy()
    for b in range(q.shape[0]):
        for l in layers:
            g, ll = divmod(l, w.layers_per_group)
            ck = cells[cell_index(w, b, g, 0)]
            cv = cells[cell_index(w, b, g, 1)]
            Kh = oracle.decompress_cell(ck, rot_seed)[ll]
            Vh = oracle.decompress_cell(cv, rot_seed)[ll]
            if w.keys_pre_rope:
                Kh = oracle.rope(Kh, pos_offset + np.arange(w.T), inv_freq)
            res[(b, l)] = oracle.decode_attention(Kh, Vh, qn[b, l], scale)
    return res


def max_rel_err(out, ref):
    """max over query-head vectors of ||o - ref||_inf / ||ref||_inf."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(out - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return float(np.max(num / den))


def device_to_cells(shape, w, cache, choices, factor_dtype=None):
    """Read a device cache (jolt layout) back into oracle cell dicts (stored values as float64)."""
    fdt = _FDT[factor_dtype or w.factor_dtype]
    esz = 4 if fdt == torch.float32 else 2
    offs, total = api.cache_layout(shape, choices)
    buf = cache.cpu()
    Lg, H, T, d = w.layers_per_group, w.n_kv, shape.T, w.d_h
    cells = []

    def get(off, count, dtype):
        raw = buf[int(off):int(off) + count * (torch.finfo(dtype).bits // 8 if dtype.is_floating_point else 1)]
        return raw.view(dtype)

    for c, (rT, rd, b) in enumerate(choices):
        cell = {"r_T": rT, "r_d": rd, "b": b, "shape": (Lg, H, T, d)}
        if rT:
            cell["U_T"] = get(offs[c, 0], T * rT, fdt).double().numpy().reshape(T, rT)
            cell["U_d"] = get(offs[c, 1], d * rd, fdt).double().numpy().reshape(d, rd)
            cell["G"] = get(offs[c, 2], Lg * H * rT * rd, fdt).double().numpy().reshape(Lg, H, rT, rd)
        else:
            cell["U_T"] = np.zeros((T, 0)); cell["U_d"] = np.zeros((d, 0)); cell["G"] = np.zeros((Lg, H, 0, 0))
        if b:
            cell["codes"] = buf[int(offs[c, 3]):int(offs[c, 3]) + Lg * H * T * d * b // 8].numpy().reshape(Lg, H, T, d * b // 8)
            sz = get(offs[c, 4], Lg * H * T * 2, torch.float16).numpy().reshape(Lg, H, T, 2)
            cell["scale"] = sz[..., 0].copy()
            cell["zero"] = sz[..., 1].copy()
        cells.append(cell)
    return cells


def device_cell(shape, w, cache, choices, c, factor_dtype=None):
    """One cell of a device cache as an oracle cell dict (only that cell's bytes are copied)."""
    fdt = _FDT[factor_dtype or w.factor_dtype]
    offs, _ = api.cache_layout(shape, choices)
    Lg, H, T, d = w.layers_per_group, w.n_kv, shape.T, w.d_h
    rT, rd, b = choices[c]

    def get(off, count, dtype):
        nb = count * (torch.finfo(dtype).bits // 8 if dtype.is_floating_point else 1)
        return cache[int(off):int(off) + nb].cpu().view(dtype)

    cell = {"r_T": rT, "r_d": rd, "b": b, "shape": (Lg, H, T, d)}
    if rT:
        cell["U_T"] = get(offs[c, 0], T * rT, fdt).double().numpy().reshape(T, rT)
        cell["U_d"] = get(offs[c, 1], d * rd, fdt).double().numpy().reshape(d, rd)
        cell["G"] = get(offs[c, 2], Lg * H * rT * rd, fdt).double().numpy().reshape(Lg, H, rT, rd)
    else:
        cell["U_T"] = np.zeros((T, 0)); cell["U_d"] = np.zeros((d, 0)); cell["G"] = np.zeros((Lg, H, 0, 0))
    if b:
        cell["codes"] = get(offs[c, 3], Lg * H * T * d * b // 8, torch.uint8).numpy().reshape(Lg, H, T, d * b // 8)
        sz = get(offs[c, 4], Lg * H * T * 2, torch.float16).numpy().reshape(Lg, H, T, 2)
        cell["scale"] = sz[..., 0].copy()
        cell["zero"] = sz[..., 1].copy()
    return cell
