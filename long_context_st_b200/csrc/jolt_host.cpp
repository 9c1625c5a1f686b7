// Host-side part of the JoLT library: shape checks, byte model, stored-cache layout, the
// quantiser error fraction phi(b), and the single-multiplier allocator.
//
// Compiled with -ffp-contract=off so that E + lambda*bytes style expressions round exactly as
// written (no fused multiply-add).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "jolt_internal.h"

namespace jolt {

bool shape_ok(const jolt_shape* s) {
  if (!s) return false;
  if (s->batch < 1 || s->n_layers < 1 || s->layers_per_group < 1 || s->n_kv < 1 || s->T < 1)
    return false;
  if (s->n_layers % s->layers_per_group) return false;
  if (s->n_q < s->n_kv || s->n_q % s->n_kv) return false;
  if (s->d_h != 64 && s->d_h != 128) return false;
  if (s->io_dtype != JOLT_F32 && s->io_dtype != JOLT_BF16) return false;
  if (s->factor_dtype != JOLT_F32 && s->factor_dtype != JOLT_BF16) return false;
  const int64_t n = n_cols(*s);
  const int64_t lim = std::min<int64_t>(n, s->T);
  if (s->q_cap < 0 || s->q_cap % kRankStep || s->q_cap > lim) return false;
  if (s->sketch_cols % kRankStep || s->sketch_cols < s->q_cap || s->sketch_cols > lim) return false;
  if (s->q_cap > 0 && s->sketch_cols < 16) return false;
  if (s->power_iters < 0 || s->power_iters > 8) return false;
  if (s->cells_per_pass < 1) return false;
  if (!(s->attn_scale > 0.f) || !std::isfinite(s->attn_scale)) return false;
  if (!std::isfinite(s->rope_attention_scaling)) return false;
  if (s->T > (1 << 24)) return false;
  if (s->gemm_plan < JOLT_GEMM_DEFAULT || s->gemm_plan > JOLT_GEMM_PAIRS) return false;
  return true;
}

bool choice_ok(const jolt_shape& s, const jolt_cell_choice& c) {
  if (c.r_T < 0 || c.r_d < 0 || c.r_T % kRankStep || c.r_d % kRankStep) return false;
  if ((c.r_T == 0) != (c.r_d == 0)) return false;
  if (c.r_T > s.q_cap || c.r_d > s.d_h) return false;
  if (!(c.b == 0 || c.b == 2 || c.b == 4 || c.b == 8)) return false;
  return true;
}

CellSegs cell_segments(const jolt_shape& s, const jolt_cell_choice& c) {
  const SegOffsets o = seg_offsets(s.T, s.d_h, s.layers_per_group, s.n_kv, dtype_bytes(s.factor_dtype),
                                   c.r_T, c.r_d, c.b);
  const uint64_t rows = uint64_t(s.layers_per_group) * s.n_kv * s.T;
  CellSegs g{o.ut, o.ud, o.g, o.codes, o.sz, 0};
  g.size = align_up(o.sz + (c.b ? rows * 4 : 0), kSegAlign);
  return g;
}

// ---- fp16 / Gaussian helpers for phi --------------------------------------------------------

static inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Standard normal pairs by the Box-Muller transform on two counter-hashed uniforms in (0, 1).
static inline void normal_pair(uint64_t seed, uint64_t i, double* a, double* b) {
  const double u1 = (double((splitmix64((seed << 32) ^ (2 * i)) >> 11)) + 0.5) * 0x1.0p-53;
  const double u2 = (double((splitmix64((seed << 32) ^ (2 * i + 1)) >> 11)) + 0.5) * 0x1.0p-53;
  const double r = std::sqrt(-2.0 * std::log(u1));
  *a = r * std::cos(6.283185307179586 * u2);
  *b = r * std::sin(6.283185307179586 * u2);
}

static inline float to_f16_and_back(float x, bool* overflow) {
  _Float16 h = (_Float16)x;  // round to nearest even
  float y = (float)h;
  if (!std::isfinite(y)) *overflow = true;
  return y;
}

}  // namespace jolt

using namespace jolt;

extern "C" {

const char* jolt_status_string(jolt_status s) {
  switch (s) {
    case JOLT_OK: return "ok";
    case JOLT_ERR_INVALID_ARG: return "invalid argument";
    case JOLT_ERR_CUDA: return "CUDA error";
    case JOLT_ERR_TIMEOUT: return "device wait timed out";
    case JOLT_ERR_BUDGET: return "byte budget infeasible";
    case JOLT_ERR_NUMERIC: return "numeric range error";
    case JOLT_ERR_WORKSPACE: return "workspace too small";
    case JOLT_ERR_STATE: return "workspace not prepared by jolt_analyze";
  }
  return "unknown status";
}

int32_t jolt_version(void) { return 100; }

jolt_status jolt_shape_check(const jolt_shape* s) {
  return shape_ok(s) ? JOLT_OK : JOLT_ERR_INVALID_ARG;
}

uint64_t jolt_kv_bytes(int32_t n_layers, int32_t n_kv, int32_t d_h, int64_t T, int32_t dtype_bytes_) {
  if (n_layers < 0 || n_kv < 0 || d_h < 0 || T < 0 || dtype_bytes_ < 0) return 0;
  return 2ull * uint64_t(n_layers) * uint64_t(n_kv) * uint64_t(d_h) * uint64_t(T) *
         uint64_t(dtype_bytes_);
}

uint64_t jolt_cell_bytes(const jolt_shape* s, jolt_cell_choice c) {
  if (!shape_ok(s) || !choice_ok(*s, c)) return 0;
  const uint64_t sf = dtype_bytes(s->factor_dtype);
  const uint64_t T = s->T, d = s->d_h, Lg = s->layers_per_group, H = s->n_kv;
  uint64_t bytes = sf * (T * c.r_T + d * c.r_d + Lg * H * uint64_t(c.r_T) * c.r_d);
  if (c.b > 0) bytes += Lg * H * T * (d * c.b / 8 + 4);
  return bytes;
}

jolt_status jolt_cache_layout(const jolt_shape* s, const jolt_cell_choice* choices,
                              uint64_t* offsets, uint64_t* total_bytes) {
  if (!shape_ok(s) || !choices || !total_bytes) return JOLT_ERR_INVALID_ARG;
  const int nc = n_cells(*s);
  uint64_t off = 0;
  for (int c = 0; c < nc; ++c) {
    if (!choice_ok(*s, choices[c])) return JOLT_ERR_INVALID_ARG;
    CellSegs g = cell_segments(*s, choices[c]);
    if (offsets) {
      offsets[5 * c + 0] = off + g.ut;
      offsets[5 * c + 1] = off + g.ud;
      offsets[5 * c + 2] = off + g.g;
      offsets[5 * c + 3] = off + g.codes;
      offsets[5 * c + 4] = off + g.sz;
    }
    off += g.size;
  }
  *total_bytes = off;
  return JOLT_OK;
}

jolt_status jolt_phi(int32_t d_h, int32_t n_rows, uint64_t seed, double phi_out[4]) {
  if (!phi_out || d_h < 2 || d_h > 4096 || n_rows < 1) return JOLT_ERR_INVALID_ARG;
  std::vector<float> row(d_h);
  double tot = 0.0, err[3] = {0.0, 0.0, 0.0};
  const int bits[3] = {2, 4, 8};
  bool ovf = false;
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int j = 0; j < d_h; j += 2) {
      double a, b;
      normal_pair(seed, uint64_t(r) * d_h + j, &a, &b);
      row[j] = float(a);
      if (j + 1 < d_h) row[j + 1] = float(b);
    }
    float mn = row[0], mx = row[0];
    for (int j = 0; j < d_h; ++j) {
      mn = std::min(mn, row[j]);
      mx = std::max(mx, row[j]);
      tot += double(row[j]) * double(row[j]);
    }
    for (int bi = 0; bi < 3; ++bi) {
      const int b = bits[bi];
      const float levels = float((1 << b) - 1);
      const float rng = mx - mn;
      const float step = rng / levels;
      const float scale = to_f16_and_back(step, &ovf);
      const float zero = to_f16_and_back(mn, &ovf);
      for (int j = 0; j < d_h; ++j) {
        float code = 0.f;
        if (scale != 0.f) {
          const float diff = row[j] - zero;
          code = std::nearbyint(diff / scale);  // default rounding mode: nearest even
          code = std::min(std::max(code, 0.f), levels);
        }
        const float deq = float(double(code) * double(scale) + double(zero));
        const double e = double(row[j]) - double(deq);
        err[bi] += e * e;
      }
    }
  }
  if (ovf) return JOLT_ERR_NUMERIC;
  phi_out[0] = 1.0;
  for (int bi = 0; bi < 3; ++bi) phi_out[bi + 1] = err[bi] / tot;
  return JOLT_OK;
}

// ---- allocator ------------------------------------------------------------------------------

namespace {
struct Opt {
  uint64_t B;
  double E;
  int rT, rd, b;
};
struct Seg {
  double price;
  int cell, idx;
  uint64_t dB;
};

double cross3(const Opt& a, const Opt& b, const Opt& c) {
  const double t1 = (double(b.B) - double(a.B)) * (c.E - a.E);
  const double t2 = (b.E - a.E) * (double(c.B) - double(a.B));
  return t1 - t2;
}
}  // namespace

jolt_status jolt_allocate(const jolt_shape* s, int32_t nc, const double* norm2,
                          const double* tail_T, int32_t nrt, const double* tail_d, int32_t nrd,
                          const double phi[4], uint64_t budget, jolt_cell_choice* out,
                          double* lambda_out, uint64_t* total_out) {
  if (!shape_ok(s) || nc < 1 || !norm2 || !tail_T || !tail_d || !phi || !out) return JOLT_ERR_INVALID_ARG;
  if (nrt < 1 || nrd < 1 || (nrt - 1) * kRankStep > s->q_cap || (nrd - 1) * kRankStep > s->d_h)
    return JOLT_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!(phi[i] >= 0.0) || !std::isfinite(phi[i])) return JOLT_ERR_INVALID_ARG;
  const int bits[4] = {0, 2, 4, 8};
  std::vector<std::vector<Opt>> hulls(nc);
  for (int c = 0; c < nc; ++c) {
    std::vector<Opt> opts;
    opts.reserve(size_t(1 + (nrt - 1) * (nrd - 1)) * 4);
    for (int k = 0; k < nrt; ++k) {
      for (int j = 0; j < nrd; ++j) {
        if ((k == 0) != (j == 0)) continue;
        if (k == 0 && j != 0) continue;
        double D;
        if (k == 0) {
          D = norm2[c];
        } else {
          const double sum = tail_T[size_t(c) * nrt + k] + tail_d[size_t(c) * nrd + j];
          D = std::min(norm2[c], sum);
        }
        if (!std::isfinite(D)) return JOLT_ERR_NUMERIC;
        for (int bi = 0; bi < 4; ++bi) {
          jolt_cell_choice ch{k * kRankStep, j * kRankStep, bits[bi]};
          Opt o;
          o.B = jolt_cell_bytes(s, ch);
          o.E = D * phi[bi];
          o.rT = ch.r_T;
          o.rd = ch.r_d;
          o.b = ch.b;
          opts.push_back(o);
        }
      }
    }
    std::sort(opts.begin(), opts.end(), [](const Opt& a, const Opt& b) {
      if (a.B != b.B) return a.B < b.B;
      if (a.E != b.E) return a.E < b.E;
      if (a.rT != b.rT) return a.rT < b.rT;
      if (a.rd != b.rd) return a.rd < b.rd;
      return a.b < b.b;
    });
    std::vector<Opt> front;
    for (const Opt& o : opts) {
      if (!front.empty() && front.back().B == o.B) continue;
      if (!front.empty() && !(o.E < front.back().E)) continue;
      front.push_back(o);
    }
    std::vector<Opt>& h = hulls[c];
    for (const Opt& o : front) {
      while (h.size() >= 2 && cross3(h[h.size() - 2], h[h.size() - 1], o) <= 0.0) h.pop_back();
      h.push_back(o);
    }
  }
  uint64_t total = 0;
  for (int c = 0; c < nc; ++c) total += hulls[c][0].B;
  if (total > budget) return JOLT_ERR_BUDGET;
  std::vector<Seg> segs;
  for (int c = 0; c < nc; ++c) {
    double prev = INFINITY;
    const auto& h = hulls[c];
    for (size_t i = 1; i < h.size(); ++i) {
      const uint64_t dB = h[i].B - h[i - 1].B;
      const double dE = h[i - 1].E - h[i].E;
      double price = dE / double(dB);
      price = std::min(price, prev);
      prev = price;
      segs.push_back(Seg{price, c, int(i), dB});
    }
  }
  std::sort(segs.begin(), segs.end(), [](const Seg& a, const Seg& b) {
    if (a.price != b.price) return a.price > b.price;
    if (a.cell != b.cell) return a.cell < b.cell;
    return a.idx < b.idx;
  });
  std::vector<int> pos(nc, 0);
  double lam = 0.0;
  for (const Seg& sg : segs) {
    if (total + sg.dB <= budget) {
      if (pos[sg.cell] != sg.idx - 1) return JOLT_ERR_NUMERIC;  // cannot happen on a valid hull
      pos[sg.cell] = sg.idx;
      total += sg.dB;
    } else {
      lam = sg.price;
      break;
    }
  }
  for (int c = 0; c < nc; ++c) {
    const Opt& o = hulls[c][pos[c]];
    out[c] = jolt_cell_choice{o.rT, o.rd, o.b};
  }
  if (lambda_out) *lambda_out = lam;
  if (total_out) *total_out = total;
  return JOLT_OK;
}

namespace {

// One option of a cell: bytes, modelled error and the choice.
struct CoordOpt {
  uint64_t B;
  double E;
  int32_t rT, rd, b;
};

// Ordering of the coordinate search: E + lam * bytes, then bytes, r_T, r_d, b.
bool coord_less(const CoordOpt& x, const CoordOpt& y, double lam) {
  const double vx = x.E + lam * double(x.B), vy = y.E + lam * double(y.B);
  if (vx != vy) return vx < vy;
  if (x.B != y.B) return x.B < y.B;
  if (x.rT != y.rT) return x.rT < y.rT;
  if (x.rd != y.rd) return x.rd < y.rd;
  return x.b < y.b;
}

// The coordinate-wise rank search of one cell at multiplier lam: from full ranks, the best r_T
// with r_d held (a zero token rank takes the residual-only options), then the best r_d with r_T
// held, b chosen with each move, until a round changes nothing (at most 32 rounds).
CoordOpt coord_cell(const std::vector<CoordOpt>& opts, int32_t rTmax, int32_t rdmax, double lam) {
  const CoordOpt* cur = nullptr;
  for (const CoordOpt& o : opts)
    if (o.rT == rTmax && o.rd == rdmax && (!cur || coord_less(o, *cur, lam))) cur = &o;
  for (int round = 0; round < 32; ++round) {
    const CoordOpt* start = cur;
    const CoordOpt* best = nullptr;
    for (const CoordOpt& o : opts)
      if ((o.rd == cur->rd || o.rT == 0) && (!best || coord_less(o, *best, lam))) best = &o;
    cur = best;
    best = nullptr;
    for (const CoordOpt& o : opts)
      if (o.rT == cur->rT && (!best || coord_less(o, *best, lam))) best = &o;
    cur = best;
    if (cur == start) break;
  }
  return *cur;
}

// Coordinate-wise allocation: the multiplier from a geometric bisection of [1e-30, 1e30] (200
// halvings, midpoint sqrt(lo * hi)); the allocation of the bracket end that fits the budget.
jolt_status allocate_coord(const jolt_shape* s, int32_t nc, const double* norm2, const double* tail_T, int32_t nrt,
                           const double* tail_d, int32_t nrd, const double phi[4], uint64_t budget,
                           jolt_cell_choice* out, uint64_t* total_out) {
  const int bits[4] = {0, 2, 4, 8};
  std::vector<std::vector<CoordOpt>> cells(nc);
  for (int c = 0; c < nc; ++c) {
    if (!std::isfinite(norm2[c])) return JOLT_ERR_NUMERIC;
    for (int k = 0; k < nrt; ++k)
      for (int j = 0; j < nrd; ++j) {
        if ((k == 0) != (j == 0)) continue;
        const double D = k == 0 ? norm2[c] : std::min(norm2[c], tail_T[size_t(c) * nrt + k] + tail_d[size_t(c) * nrd + j]);
        if (!std::isfinite(D)) return JOLT_ERR_NUMERIC;
        for (int bi = 0; bi < 4; ++bi) {
          const jolt_cell_choice ch{k * kRankStep, j * kRankStep, bits[bi]};
          cells[c].push_back(CoordOpt{jolt_cell_bytes(s, ch), D * phi[bi], ch.r_T, ch.r_d, ch.b});
        }
      }
  }
  const int32_t rTmax = (nrt - 1) * kRankStep, rdmax = (nrd - 1) * kRankStep;
  std::vector<CoordOpt> pick(nc), best(nc);
  auto at = [&](double lam, std::vector<CoordOpt>& dst) {
    uint64_t tot = 0;
    for (int c = 0; c < nc; ++c) {
      dst[c] = coord_cell(cells[c], rTmax, rdmax, lam);
      tot += dst[c].B;
    }
    return tot;
  };
  double lo = 1e-30, hi = 1e30;
  uint64_t b_hi = at(hi, best);
  if (b_hi > budget) return JOLT_ERR_BUDGET;
  uint64_t b_lo = at(lo, pick);
  if (b_lo <= budget) {
    best = pick;
    b_hi = b_lo;
  } else {
    for (int it = 0; it < 200; ++it) {
      const double mid = std::sqrt(lo * hi);
      const uint64_t b = at(mid, pick);
      if (b <= budget) {
        hi = mid;
        best = pick;
        b_hi = b;
      } else {
        lo = mid;
      }
    }
  }
  for (int c = 0; c < nc; ++c) out[c] = jolt_cell_choice{best[c].rT, best[c].rd, best[c].b};
  if (total_out) *total_out = b_hi;
  return JOLT_OK;
}

}  // namespace

jolt_status jolt_allocate_variant(const jolt_shape* s, int32_t nc, const double* norm2, const double* tail_T,
                                  int32_t nrt, const double* tail_d, int32_t nrd, const double phi[4],
                                  uint64_t budget, int32_t mode, jolt_cell_choice* out, uint64_t* total_out) {
  if (mode == JOLT_ALLOC_JOINT)
    return jolt_allocate(s, nc, norm2, tail_T, nrt, tail_d, nrd, phi, budget, out, nullptr, total_out);
  if (!shape_ok(s) || nc < 2 || nc % 2 || !norm2 || !tail_T || !tail_d || !phi || !out) return JOLT_ERR_INVALID_ARG;
  if (nrt < 1 || nrd < 1 || (nrt - 1) * kRankStep > s->q_cap || (nrd - 1) * kRankStep > s->d_h)
    return JOLT_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!(phi[i] >= 0.0) || !std::isfinite(phi[i])) return JOLT_ERR_INVALID_ARG;
  const int half = nc / 2;
  if (mode == JOLT_ALLOC_KV_SPLIT) {
    uint64_t total = 0;
    for (int kind = 0; kind < 2; ++kind) {
      std::vector<double> n2(half), tT(size_t(half) * nrt), td(size_t(half) * nrd);
      for (int i = 0; i < half; ++i) {
        const int c = 2 * i + kind;
        n2[i] = norm2[c];
        std::copy(tail_T + size_t(c) * nrt, tail_T + size_t(c + 1) * nrt, tT.begin() + size_t(i) * nrt);
        std::copy(tail_d + size_t(c) * nrd, tail_d + size_t(c + 1) * nrd, td.begin() + size_t(i) * nrd);
      }
      std::vector<jolt_cell_choice> ch(half);
      uint64_t tot = 0;
      const uint64_t bud = kind == 0 ? budget / 2 : budget - budget / 2;
      const jolt_status r = jolt_allocate(s, half, n2.data(), tT.data(), nrt, td.data(), nrd, phi, bud, ch.data(),
                                          nullptr, &tot);
      if (r != JOLT_OK) return r;
      for (int i = 0; i < half; ++i) out[2 * i + kind] = ch[i];
      total += tot;
    }
    if (total_out) *total_out = total;
    return JOLT_OK;
  }
  if (mode == JOLT_ALLOC_COORD) return allocate_coord(s, nc, norm2, tail_T, nrt, tail_d, nrd, phi, budget, out, total_out);
  if (mode != JOLT_ALLOC_UNIFORM) return JOLT_ERR_INVALID_ARG;
  // every choice in (r_T, r_d, b) order with its bytes and its summed error over each kind's cells
  const int bits[4] = {0, 2, 4, 8};
  std::vector<jolt_cell_choice> grid;
  for (int k = 0; k < nrt; ++k)
    for (int j = 0; j < nrd; ++j) {
      if ((k == 0) != (j == 0)) continue;
      for (int bi = 0; bi < 4; ++bi) grid.push_back(jolt_cell_choice{k * kRankStep, j * kRankStep, bits[bi]});
    }
  const size_t ng = grid.size();
  std::vector<uint64_t> gb(ng);
  std::vector<double> ge[2] = {std::vector<double>(ng, 0.0), std::vector<double>(ng, 0.0)};
  for (size_t o = 0; o < ng; ++o) {
    const jolt_cell_choice& ch = grid[o];
    gb[o] = jolt_cell_bytes(s, ch);
    const int k = ch.r_T / kRankStep, j = ch.r_d / kRankStep;
    const int bi = ch.b == 0 ? 0 : ch.b == 2 ? 1 : ch.b == 4 ? 2 : 3;
    for (int c = 0; c < nc; ++c) {
      const double D = k == 0 ? norm2[c] : std::min(norm2[c], tail_T[size_t(c) * nrt + k] + tail_d[size_t(c) * nrd + j]);
      if (!std::isfinite(D)) return JOLT_ERR_NUMERIC;
      ge[c % 2][o] += D * phi[bi];
    }
  }
  bool found = false;
  double bestE = 0.0;
  uint64_t bestB = 0;
  size_t bk = 0, bv = 0;
  for (size_t ok = 0; ok < ng; ++ok) {
    const uint64_t bK = uint64_t(half) * gb[ok];
    if (bK > budget) continue;
    for (size_t ov = 0; ov < ng; ++ov) {
      const uint64_t B = bK + uint64_t(half) * gb[ov];
      if (B > budget) continue;
      const double E = ge[0][ok] + ge[1][ov];
      if (!found || E < bestE || (E == bestE && B < bestB)) {
        found = true;
        bestE = E;
        bestB = B;
        bk = ok;
        bv = ov;
      }
    }
  }
  if (!found) return JOLT_ERR_BUDGET;
  for (int c = 0; c < nc; ++c) out[c] = grid[c % 2 ? bv : bk];
  if (total_out) *total_out = bestB;
  return JOLT_OK;
}

size_t jolt_workspace_bytes(const jolt_shape* s, int32_t op) {
  if (!shape_ok(s)) return 0;
  if (op == JOLT_OP_COMPRESS) return compress_workspace_bytes(*s);
  if (op == JOLT_OP_DECODE) return decode_workspace_bytes(*s);
  return 0;
}

}  // extern "C"

extern "C" jolt_status jolt_group_layers(const double* align, int32_t n_layers, double tau, int32_t max_group,
                                         int32_t* group_sizes, int32_t* n_groups) {
  if (n_layers < 1 || !group_sizes || !n_groups || (n_layers > 1 && !align)) return JOLT_ERR_INVALID_ARG;
  int ng = 1;
  group_sizes[0] = 1;
  for (int l = 0; l + 1 < n_layers; ++l) {
    if (align[l] >= tau && (max_group <= 0 || group_sizes[ng - 1] < max_group)) {
      ++group_sizes[ng - 1];
    } else {
      group_sizes[ng++] = 1;
    }
  }
  *n_groups = ng;
  return JOLT_OK;
}

extern "C" jolt_status jolt_uniform_group(const double* align, int32_t n_layers, double tau, int32_t* L_g) {
  if (n_layers < 1 || !L_g || (n_layers > 1 && !align)) return JOLT_ERR_INVALID_ARG;
  int best = 1;
  for (int g = 1; g <= n_layers; ++g) {
    if (n_layers % g) continue;
    bool ok = true;
    for (int l = 0; l + 1 < n_layers && ok; ++l)
      if ((l + 1) % g != 0 && !(align[l] >= tau)) ok = false;
    if (ok) best = g;
  }
  *L_g = best;
  return JOLT_OK;
}
