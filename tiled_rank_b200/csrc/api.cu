// C ABI of the TileQ MoE forward (include/tileq.h): host-side validation,
// packed-weight and workspace layouts, the per-GEMM launch plan, and the
// launch sequence of the fused and of the unfused (per-expert) forward.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "kernels.cuh"

using namespace tileq;

namespace tileq {
void count_launches(int n);
}

namespace {

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }
int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }
unsigned nblocks(long long n, int per) { return (unsigned)((n + per - 1) / per); }

constexpr int kNumSMs = 148;
// gather_ext_kernel: one chunk per thread while that fits in one wave of CTAs
// (short batches: the z sums need the parallelism), then grid-stride with
// kGatherUnroll chunks per thread in flight
unsigned gather_blocks(long long chunks) {
  return std::max(1u, std::min(nblocks(chunks, 256), 8u * kNumSMs));
}
// split the narrow residual GEMM until ~this many CTAs per SM
constexpr int kQ2PerSm = 4;
constexpr int kTcMinTokens = 256;  // dense fp16 products (z, shared expert) move to tcgen05 from here
constexpr int kWideMinK = 4096;    // 256-item tcgen05 tiles from this K (32 stages per unit) on

struct ProjInfo {
  int d_in, d_out, rank, group, G;
  int bits;   // 2 or 3
  int8_t m_of[kMaxExperts], n_of[kMaxExperts];
};

struct LayerInfo {
  int nproj, K;
  ProjInfo p[3];
  int d_x, d_y;
};

tileq_status validate_layer(const tileq_layer *L, LayerInfo *li, bool need_device_ptrs = true) {
  if (!L) return TILEQ_ERR_INVALID_ARG;
  if (L->kind != TILEQ_LINEAR && L->kind != TILEQ_SWIGLU) return TILEQ_ERR_INVALID_ARG;
  if (L->route_mode != TILEQ_ROUTE_TOPK_SOFTMAX && L->route_mode != TILEQ_ROUTE_FULL_SOFTMAX)
    return TILEQ_ERR_INVALID_ARG;
  if (L->K < 1 || L->M < 1 || L->N < 1 || (long long)L->M * L->N < L->K) return TILEQ_ERR_INVALID_ARG;
  if (L->K > kMaxExperts || L->M > kMaxExperts || L->N > kMaxExperts) return TILEQ_ERR_UNSUPPORTED;
  li->nproj = L->kind == TILEQ_LINEAR ? 1 : 3;
  li->K = L->K;
  for (int pi = 0; pi < li->nproj; ++pi) {
    const tileq_proj &p = L->proj[pi];
    ProjInfo &q = li->p[pi];
    if (p.d_in <= 0 || p.d_out <= 0 || p.rank < 0 || p.group <= 0) return TILEQ_ERR_INVALID_ARG;
    if (p.bits != 0 && p.bits != 2 && p.bits != 3) return TILEQ_ERR_UNSUPPORTED;
    if (p.d_out % 16 || p.d_in % 128 || (p.group != 64 && p.group % 128) || p.d_in % p.group ||
        p.rank % 16 ||
        p.rank > 256)
      return TILEQ_ERR_UNSUPPORTED;
    if (!p.grid_assign) return TILEQ_ERR_INVALID_ARG;
    if (need_device_ptrs) {
      if (!p.codes || !p.scales || !p.zeros) return TILEQ_ERR_INVALID_ARG;
      if (p.bits == 3 && !p.codes_hi) return TILEQ_ERR_INVALID_ARG;
      if (p.rank > 0 && (!p.U || !p.V || !p.Sigma)) return TILEQ_ERR_INVALID_ARG;
    }
    std::vector<char> seen((size_t)L->M * L->N, 0);
    for (int e = 0; e < L->K; ++e) {
      const int cell = p.grid_assign[e];
      if (cell < 0 || cell >= L->M * L->N || seen[cell]) return TILEQ_ERR_INVALID_ARG;
      seen[cell] = 1;
      q.m_of[e] = (int8_t)(cell / L->N);
      q.n_of[e] = (int8_t)(cell % L->N);
    }
    q.d_in = p.d_in;
    q.d_out = p.d_out;
    q.rank = p.rank;
    q.group = p.group;
    q.G = p.d_in / p.group;
    q.bits = p.bits == 3 ? 3 : 2;
  }
  if (L->kind == TILEQ_SWIGLU) {
    const ProjInfo &g = li->p[0], &u = li->p[1], &d = li->p[2];
    if (g.d_in != L->d_model || g.d_out != L->d_ff || u.d_in != L->d_model || u.d_out != L->d_ff ||
        d.d_in != L->d_ff || d.d_out != L->d_model)
      return TILEQ_ERR_INVALID_ARG;
    if (g.rank != u.rank) return TILEQ_ERR_UNSUPPORTED;
    if (g.bits != u.bits) return TILEQ_ERR_UNSUPPORTED;   // gate and up share one residual kernel
    if (L->shared_d_ff < 0) return TILEQ_ERR_INVALID_ARG;
    if (L->shared_d_ff > 0) {
      if (L->shared_d_ff % 128) return TILEQ_ERR_UNSUPPORTED;
      if (need_device_ptrs && (!L->shared_w[0] || !L->shared_w[1] || !L->shared_w[2]))
        return TILEQ_ERR_INVALID_ARG;
    }
  } else if (L->shared_d_ff != 0) {
    return TILEQ_ERR_INVALID_ARG;
  }
  li->d_x = li->p[0].d_in;
  li->d_y = li->p[li->nproj - 1].d_out;
  return TILEQ_OK;
}

// ------------------------------------------------------------------ packed layouts
size_t frag_bytes(int nblk, int R, int C, int kb) {
  return (size_t)nblk * pad128(R) * (size_t)cdiv(C, 16 * kb) * 16 * kb * 2;
}

// qw: codes in the row layout of the tcgen05 kernel; qf: the same codes in the
// per-lane A-fragment order of the warp-MMA streaming kernel.
// sig: Sigma repeated per grid column ([N][pad128(rank)] fp32), the column
// scales of the projection onto all grid columns at once.  vr: V_n^T rows in
// fp16, row-major [N][pad128(rank)][d_in], and shr: the shared expert's
// weights row-major fp16 [pad128(rows)][cols] (the A operands of the tcgen05
// kernel; vf / sh hold the same values in warp-MMA fragment order).
struct PackedLayout {
  size_t qw[3], qwh[3], qf[3], qfh[3], sz[3], uf[3], vf[3], sig[3], vr[3], sh[3], shr[3], total;
};

PackedLayout packed_layout(const tileq_layer *L, const LayerInfo &li) {
  PackedLayout pl{};
  size_t off = 0;
  for (int p = 0; p < li.nproj; ++p) {
    const ProjInfo &q = li.p[p];
    pl.qw[p] = off;   // tcgen05 row layout
    off += align_up((size_t)L->K * pad128(q.d_out) * q.d_in / 4);
    pl.qwh[p] = off;  // 3-bit high-bit plane, row layout
    if (q.bits == 3) off += align_up((size_t)L->K * pad128(q.d_out) * q.d_in / 8);
    pl.qf[p] = off;
    off += align_up((size_t)L->K * pad128(q.d_out) * q.d_in / 4);
    pl.qfh[p] = off;  // 3-bit high-bit plane, fragment layout
    if (q.bits == 3) off += align_up((size_t)L->K * pad128(q.d_out) * q.d_in / 8);
    pl.sz[p] = off;
    off += align_up((size_t)L->K * pad128(q.d_out) * q.G * 4);
    pl.uf[p] = off;
    if (q.rank > 0) off += align_up((size_t)L->M * pad128(q.d_out) * q.rank * 2);
    pl.vf[p] = off;
    if (q.rank > 0) off += align_up(frag_bytes(L->N, q.rank, q.d_in, 8));
    pl.sig[p] = off;
    if (q.rank > 0) off += align_up((size_t)L->N * pad128(q.rank) * 4);
    pl.vr[p] = off;
    if (q.rank > 0) off += align_up((size_t)L->N * pad128(q.rank) * q.d_in * 2);
  }
  for (int i = 0; i < 3; ++i) {
    pl.sh[i] = off;
    pl.shr[i] = off;
    if (L->shared_d_ff > 0) {
      const int R = i < 2 ? L->shared_d_ff : L->d_model, C = i < 2 ? L->d_model : L->shared_d_ff;
      off += align_up(frag_bytes(1, R, C, 8));
      pl.shr[i] = off;
      off += align_up((size_t)pad128(R) * C * 2);
    }
  }
  pl.total = off;
  return pl;
}

// Per-expert factors of the unfused comparison path: warp-MMA fragment order
// (uf, vf) for short batches and row-major fp16 (ur = U_pe rows
// [K][pad128(d_out)][rank], vr = V_pe^T rows [K][pad128(rank)][d_in]) for the
// dense tcgen05 kernel on long ones, the same split as the fused path.
struct PePackedLayout {
  size_t uf[3], vf[3], ur[3], vr[3], total;
};

PePackedLayout pe_layout(const tileq_layer *L, const LayerInfo &li) {
  PePackedLayout pl{};
  size_t off = 0;
  for (int p = 0; p < li.nproj; ++p) {
    const ProjInfo &q = li.p[p];
    pl.uf[p] = off;
    if (q.rank > 0) off += align_up(frag_bytes(L->K, q.d_out, q.rank, 8));
    pl.vf[p] = off;
    if (q.rank > 0) off += align_up(frag_bytes(L->K, q.rank, q.d_in, 8));
    pl.ur[p] = off;
    if (q.rank > 0) off += align_up((size_t)L->K * pad128(q.d_out) * q.rank * 2);
    pl.vr[p] = off;
    if (q.rank > 0) off += align_up((size_t)L->K * pad128(q.rank) * q.d_in * 2);
  }
  pl.total = off;
  return pl;
}

// ------------------------------------------------------------------ launch plan
struct GemmPlan {
  int bn = 8, slots = 0, ksplit = 1, m_tiles = 1, np = 1, items = 0;
  bool tc = false;       // residual GEMM on tcgen05 (wide tiles) rather than warp-level MMA
  bool q2 = false;       // residual GEMM on warp-level MMA (narrow tiles)
  bool partial = false;  // K splits store their own partials (EPI_PARTIAL_F32); no reduction scratch
  bool wide = false;     // items from the wide tile table (tiles of Plan::bn_wide)
  bool dq = false;       // residual GEMM on the decode-regime tcgen05 kernel (gemm_dq.cu, stream-K)
  bool row_pair = false; // one projection on the two-projection tcgen05 kernel, two row blocks per unit
  size_t part_floats() const {
    if (dq) return (size_t)dq_grid() * 2 * np * bn * kRowsPerCta;
    if (partial) return 0;
    // q2: one [np][bn][128] fp32 partial per (split, tile slot, row block)
    if (q2) return ksplit > 1 ? (size_t)ksplit * slots * m_tiles * np * bn * kRowsPerCta : 0;
    return ksplit > 1 ? (size_t)ksplit * np * std::max(items, 1) * m_tiles * kRowsPerCta : 0;
  }
  int counters(int nprob) const {
    if (dq) return slots * m_tiles;  // one per (tile, row block) unit
    return ksplit > 1 && !partial ? nprob * slots * m_tiles : 0;
  }
};

int choose_bn(long long avg) {
  if (avg <= 8) return 8;
  if (avg <= 16) return 16;
  if (avg <= 32) return 32;
  return 64;
}

// Items per tile of the decode-regime tcgen05 GEMM: wide enough that most
// experts fit one tile (an expert spilling into a second tile streams its
// weights twice).
int choose_bn_dq(long long avg) { return avg <= 6 ? 16 : 32; }

// Items per tile of the tensor-core GEMM (N of one tcgen05.mma: 16..128).
int choose_bn_tc(long long avg) {
  if (avg <= 16) return 16;
  if (avg <= 32) return 32;
  if (avg <= 64) return 64;
  return 128;
}

// Split K until the grid covers about `per_sm` CTAs (or work items) per SM,
// keeping >= 2 k-blocks per split.
int choose_ksplit(long long ctas, int d_in, int per_sm = 4, int cap = 8) {
  const int nkb = cdiv(d_in, 128);
  int ks = (int)std::max(1LL, ((long long)per_sm * kNumSMs + ctas - 1) / std::max(1LL, ctas));
  ks = std::min(ks, std::max(1, nkb / 2));
  return std::max(1, std::min(ks, cap));
}

struct Plan {
  int T, k, P;
  int bn_main, slots_main;
  int bn_wide = 0, slots_wide = 0;  // second tile table (one-projection tcgen05 GEMMs over long K)
  GemmPlan zproj, gateup, zdown, down, linear, sh_gu, sh_down;
  // unfused comparison path: the per-expert z products (gate/up or linear, and
  // down) and the U-side products, grouped over all experts' tiles like the
  // fused path's own projections (split-K below 256 tokens, tcgen05 above)
  GemmPlan pe_zx, pe_zd, pe_u;
};

Plan make_plan(const tileq_layer *L, const LayerInfo &li, int T, int k) {
  Plan pl;
  pl.T = T;
  pl.k = k;
  pl.P = T * k;
  const int P = pl.P;
  // Narrow tiles (<= 32 tokens per expert on average) run faster on warp-level
  // MMA than on tcgen05 (measured: an M=128 N=16 tcgen05.mma does fewer MACs per
  // cycle than mma.sync, and the decode then dominates); wider ones on tcgen05.
  const long long avg = P / std::max(1, L->K);
  const bool use_tc = avg > 32;
  // Narrow tiles run on warp-level MMA.  The decode-regime tcgen05 kernel
  // (2-bit codes in groups of a multiple of 128) is measured slower at every
  // decode shape: its per-round pipeline synchronisation outweighs the tensor
  // core rate at N <= 32, so it runs only when TILEQ_DECODE_TC=1 asks for it.
  static const bool dq_requested = [] {
    const char *v = std::getenv("TILEQ_DECODE_TC");
    return v != nullptr && v[0] == '1';
  }();
  bool dq_ok = !use_tc && dq_requested;
  for (int p = 0; p < li.nproj; ++p) dq_ok = dq_ok && li.p[p].bits == 2 && li.p[p].group % 128 == 0;
  if (dq_ok) {
    const int bn = choose_bn_dq(avg), slots = cdiv(P, bn) + L->K;
    for (int p = 0; p < li.nproj; ++p)
      dq_ok = dq_ok && dq_fits(slots, cdiv(li.p[p].d_out, 128), li.p[p].d_in, li.p[p].rank);
  }
  pl.bn_main = use_tc ? choose_bn_tc(avg) : (dq_ok ? choose_bn_dq(avg) : choose_bn(avg));
  pl.slots_main = cdiv(P, pl.bn_main) + L->K;
  const long long est_main = std::min(L->K, P) + P / pl.bn_main;
  auto tc_plan = [&](int d_out, int d_in, int np) {
    GemmPlan g;
    g.tc = use_tc;
    g.bn = pl.bn_main;
    g.slots = pl.slots_main;
    g.m_tiles = cdiv(d_out, 128);
    g.np = np;
    g.items = P;
    // tcgen05: persistent CTAs walk (tile, row block, split) items; warp MMA: one CTA each
    g.q2 = !use_tc && !dq_ok;
    g.dq = dq_ok;
    g.ksplit = dq_ok ? 1 : choose_ksplit(est_main * g.m_tiles, d_in, use_tc ? 2 : kQ2PerSm);
    return g;
  };
  // One-projection tcgen05 GEMMs over a long K take 256-item tiles (N = 256:
  // half the MMA instructions and barrier rounds per FLOP of N = 128); the
  // accumulator then fills half of tensor memory, so the epilogue no longer
  // overlaps the next unit, which only pays off when a unit spans many stages.
  auto widen = [&](GemmPlan &g, int d_in) {
    if (!use_tc || pl.bn_main != 128 || d_in < kWideMinK) return;
    pl.bn_wide = 256;
    pl.slots_wide = cdiv(P, 256) + L->K;
    g.wide = true;
    g.bn = 256;
    g.slots = pl.slots_wide;
    g.ksplit = choose_ksplit(((long long)std::min(L->K, P) + P / 256) * g.m_tiles, d_in, 2);
  };
  // A one-projection tcgen05 GEMM over a short K that is not widened runs as
  // row pairs: two 128-row blocks of the projection share each activation
  // tile (half the activation reads per FLOP) and each barrier round of the
  // MMA warp covers twice the tensor work.
  auto pair_rows = [&](GemmPlan &g, int d_out) {
    if (!g.tc || g.wide || g.ksplit != 1 || pl.bn_main != 128 || d_out <= 128) return;
    g.row_pair = true;
    g.m_tiles = cdiv(d_out, 256);
  };
  const ProjInfo &q0 = li.p[0];
  if (L->kind == TILEQ_LINEAR) {
    pl.linear = tc_plan(q0.d_out, q0.d_in, 1);
    widen(pl.linear, q0.d_in);
    pair_rows(pl.linear, q0.d_out);
  } else {
    pl.gateup = tc_plan(L->d_ff, L->d_model, 2);
    pl.down = tc_plan(L->d_model, L->d_ff, 1);
    widen(pl.down, L->d_ff);
    pair_rows(pl.down, L->d_model);
    if (li.p[2].rank > 0) {
      GemmPlan z;
      z.bn = pl.bn_main;
      z.slots = pl.slots_main;
      z.m_tiles = cdiv(li.p[2].rank, 128);
      z.items = P;
      z.ksplit = choose_ksplit(est_main * z.m_tiles, L->d_ff, 4, 16);
      // K splits reduced by the last CTA of a tile, which writes z' in fp16
      // straight into the K-extension columns of the down GEMM's activations
      z.partial = false;
      if (use_tc) {  // wide tiles: the same product on tcgen05, no K split
        z.tc = true;
        z.ksplit = 1;
      }
      pl.zdown = z;
    }
  }
  if (q0.rank > 0) {
    // z = Sigma*(V_n^T x_t) for every token and grid column: one dense product
    // [T, d_in] x [d_in, N*rank] (TileQ paper, section 2.2: the projected [T, N, r] tensor)
    GemmPlan z;
    z.bn = choose_bn(T);
    z.slots = cdiv(T, z.bn);
    z.m_tiles = L->N * (pad128(q0.rank) / 128);
    z.items = T;
    z.ksplit = choose_ksplit((long long)z.slots * z.m_tiles * (L->kind == TILEQ_SWIGLU ? 2 : 1), q0.d_in, 4, 16);
    z.partial = true;
    if (T >= kTcMinTokens) {  // long batches: tcgen05, 128-token tiles, no K split
      z.tc = true;
      z.bn = choose_bn_tc(T);
      z.slots = cdiv(T, z.bn);
      z.ksplit = 1;
    }
    pl.zproj = z;
  }
  if (L->shared_d_ff > 0) {
    const int bn = choose_bn(T);
    GemmPlan g;
    g.bn = bn;
    g.slots = cdiv(T, bn);
    g.items = T;
    g.np = 2;
    g.m_tiles = cdiv(L->shared_d_ff, 128);
    g.ksplit = choose_ksplit((long long)g.slots * g.m_tiles, L->d_model);
    pl.sh_gu = g;
    g.np = 1;
    g.m_tiles = cdiv(L->d_model, 128);
    g.ksplit = choose_ksplit((long long)g.slots * g.m_tiles, L->shared_d_ff);
    pl.sh_down = g;
    if (T >= kTcMinTokens) {  // long batches: both products on tcgen05, no K split
      for (GemmPlan *q : {&pl.sh_gu, &pl.sh_down}) {
        q->tc = true;
        q->bn = choose_bn_tc(T);
        q->slots = cdiv(T, q->bn);
        q->ksplit = 1;
      }
    }
  }
  auto pe_plan = [&](int rank, int d_in, int np) {
    GemmPlan g;
    g.bn = pl.bn_main;
    g.slots = pl.slots_main;
    g.items = P;
    g.np = np;
    g.m_tiles = std::max(1, cdiv(rank, 128));
    g.tc = T >= kTcMinTokens;
    g.ksplit = g.tc ? 1 : choose_ksplit(est_main * g.m_tiles * np, d_in, 4, 16);
    return g;
  };
  pl.pe_zx = pe_plan(q0.rank, q0.d_in, L->kind == TILEQ_SWIGLU ? 2 : 1);
  if (L->kind == TILEQ_SWIGLU) pl.pe_zd = pe_plan(li.p[2].rank, L->d_ff, 1);
  pl.pe_u = pe_plan(0, 128, 1);
  pl.pe_u.ksplit = 1;
  return pl;
}

// ------------------------------------------------------------------ workspace layout
struct WsLayout {
  Plan plan;
  size_t status, topk_idx, topk_w, expert_offsets, sorted_pairs, slot_of_pair, slot_tok, slot_w,
      dest, pcounts, tiles_main, tiles_wide, tile_first, tile_counts, counters, part;
  size_t counters_sh, part_sh;  // split-K regions of the shared expert (it runs on a side stream)
  int n_counters;
  size_t part_zstride;
  size_t zidx[2];
  size_t aidx;
  size_t x16, xext, hext, zc[2], zs, ybuf, hs, ys, g32, u32, zpe[2];
  size_t tokcnt;
  size_t x8, xs;
  int ld_x, ld_h;
  size_t total;
};

// route_only: the routing and permutation arrays alone (tileq_route and
// tileq_route_static); no GEMM scratch, no activation matrices.
WsLayout ws_layout(const tileq_layer *L, const LayerInfo &li, int T, int k, bool route_only = false) {
  WsLayout w{};
  w.plan = make_plan(L, li, T, k);
  const Plan &pl = w.plan;
  const int P = pl.P;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(std::max<size_t>(bytes, 16));
    return o;
  };
  const size_t Pz = (size_t)std::max(P, 1);
  w.status = take(256);
  w.topk_idx = take(Pz * 4);
  w.topk_w = take(Pz * 4);
  w.expert_offsets = take((L->K + 1) * 4);
  w.sorted_pairs = take(Pz * 4);
  w.slot_of_pair = take(Pz * 4);
  w.slot_tok = take(Pz * 4);
  w.slot_w = take(Pz * 4);
  w.dest = take(Pz * 4);
  w.pcounts = take((size_t)cdiv(P, kPermChunk) * L->K * 4);
  w.tiles_main = take((size_t)(pl.slots_main + 1) * 16);
  w.tiles_wide = take((size_t)(pl.slots_wide + 1) * 16);
  w.tile_first = take((L->K + 1) * 4);
  w.tile_counts = take(16);
  if (route_only) {
    w.n_counters = 0;
    w.counters = take(16);
    w.part = take(16);
    for (int z = 0; z < 2; ++z) w.zidx[z] = take(Pz * 4);
    w.aidx = take(Pz * 4);
    w.total = off;
    return w;
  }
  int nc = 0;
  nc = std::max(nc, pl.zproj.counters(2));
  nc = std::max(nc, pl.gateup.counters(1));
  nc = std::max(nc, pl.zdown.counters(1));
  nc = std::max(nc, pl.down.counters(1));
  nc = std::max(nc, pl.linear.counters(1));
  nc = std::max(nc, pl.sh_gu.counters(1));
  nc = std::max(nc, pl.sh_down.counters(1));
  nc = std::max(nc, pl.pe_zx.counters(pl.pe_zx.np));
  nc = std::max(nc, pl.pe_zd.counters(1));
  // + one arrival count per (token, output row block) for the combine fused
  // into the decode-regime down GEMM
  const int ntok = (pl.down.dq || pl.linear.dq) ? std::max(T, 1) * cdiv(li.d_y, 128) : 0;
  // + the shared expert's own counts: it runs beside the routed GEMMs
  const int nsh = L->shared_d_ff > 0 ? std::max(pl.sh_gu.counters(1), pl.sh_down.counters(1)) : 0;
  w.n_counters = nc + ntok + nsh;
  w.counters = take((size_t)(nc + ntok + nsh) * 4);
  w.tokcnt = w.counters + (size_t)nc * 4;
  w.counters_sh = w.tokcnt + (size_t)ntok * 4;
  size_t pf = 2 * pl.zproj.part_floats();
  w.part_zstride = pl.zproj.part_floats();
  for (const GemmPlan *g : {&pl.gateup, &pl.zdown, &pl.down, &pl.linear, &pl.sh_gu, &pl.sh_down, &pl.pe_zx,
                            &pl.pe_zd})
    pf = std::max(pf, g->part_floats());
  w.part = take(pf * 4);
  w.part_sh = L->shared_d_ff > 0 ? take(std::max(pl.sh_gu.part_floats(), pl.sh_down.part_floats()) * 4) : w.part;
  for (int z = 0; z < 2; ++z) w.zidx[z] = take(Pz * 4);
  w.aidx = take(Pz * 4);
  w.x16 = take((size_t)std::max(T, 1) * li.d_x * 2);
  const int rmax = std::max(std::max(li.p[0].rank, li.nproj > 1 ? li.p[1].rank : 0),
                            li.p[li.nproj - 1].rank);
  if (L->kind == TILEQ_LINEAR) {
    w.ld_x = li.d_x + li.p[0].rank;
    w.xext = take(Pz * w.ld_x * 2);
    w.zc[0] = take((size_t)pl.zproj.ksplit * std::max(T, 1) * L->N * pad128(li.p[0].rank) * 4);
  } else {
    w.ld_x = L->d_model + 2 * li.p[0].rank;
    w.ld_h = L->d_ff + li.p[2].rank;
    w.xext = take(Pz * w.ld_x * 2);
    w.hext = take(Pz * w.ld_h * 2);
    if (pl.gateup.dq) {  // e4m3 pieces of x per slot and the per-slot scales
      w.x8 = take(Pz * 2 * L->d_model);
      w.xs = take(Pz * 4);
    }
    // z for all tokens and columns, and z' per slot: fp32 partials, one per K split
    w.zc[0] = take((size_t)pl.zproj.ksplit * std::max(T, 1) * L->N * pad128(li.p[0].rank) * 4);
    w.zc[1] = take((size_t)pl.zproj.ksplit * std::max(T, 1) * L->N * pad128(li.p[1].rank) * 4);
    w.g32 = take(Pz * L->d_ff * 4);
    w.u32 = take(Pz * L->d_ff * 4);
  }
  w.zpe[0] = take(Pz * std::max(rmax, 16) * 2);
  w.zpe[1] = take(Pz * std::max(rmax, 16) * 2);
  w.ybuf = take(Pz * li.d_y * 4);
  if (L->shared_d_ff > 0) {
    w.hs = take((size_t)std::max(T, 1) * L->shared_d_ff * 2);
    w.ys = take((size_t)std::max(T, 1) * L->d_model * 4);
  }
  w.total = off;
  return w;
}

template <typename Tp>
Tp *at(void *base, size_t off) {
  return reinterpret_cast<Tp *>(static_cast<char *>(base) + off);
}
template <typename Tp>
const Tp *at(const void *base, size_t off) {
  return reinterpret_cast<const Tp *>(static_cast<const char *>(base) + off);
}

#define TQ_CUDA(call)                                 \
  do {                                                \
    if ((call) != cudaSuccess) return TILEQ_ERR_CUDA; \
  } while (0)

#define TQ_LAUNCHED()                                             \
  do {                                                            \
    count_launches();                                             \
    if (cudaGetLastError() != cudaSuccess) return TILEQ_ERR_CUDA; \
  } while (0)

std::atomic<unsigned long long> g_launches{0};
cudaEvent_t g_stage_events[16];
int g_n_stage_events = 0;

// Stage boundaries of one forward (see tileq_set_stage_events).
enum Stage { ST_BEGIN = 0, ST_ROUTE, ST_PERMUTE, ST_ZPROJ, ST_GATEUP, ST_ZDOWN, ST_SHARED, ST_RESIDUAL,
             ST_COMBINE };

void mark(int stage, cudaStream_t stream) {
  if (stage < g_n_stage_events) cudaEventRecord(g_stage_events[stage], stream);
}

// A GEMM problem with the plan's tiling and the workspace's split-K scratch.
GemmProblem problem(const GemmPlan &g, void *ws, const WsLayout &w) {
  GemmProblem p;
  std::memset(&p, 0, sizeof(p));
  p.only_group = -1;
  p.ksplit = g.ksplit;
  p.m_tiles = g.m_tiles;
  p.part = at<float>(ws, w.part);
  p.part_items = std::max(g.items, 1);
  p.counters = at<int>(ws, w.counters);
  p.status = at<int>(ws, w.status);
  return p;
}

tileq_status gemm(const GemmBatch &b, int nprob, int np, const GemmPlan &g, cudaStream_t s) {
  if (launch_gemm(b, nprob, GemmShape{np, g.bn}, g.slots, s) != cudaSuccess)
    return TILEQ_ERR_CUDA;
  return TILEQ_OK;
}

// 2-D tensor map over an fp16 matrix [rows][ld] (ld >= cols), box 64 x box_rows,
// 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap *m, const void *base, int rows, int cols, int ld, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)std::max(rows, 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map over a byte matrix [rows][cols] (row stride cols bytes, a
// multiple of 16), box 128 x box_rows, 128-byte swizzle, zero fill outside.
bool make_map_u8(CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)std::max(rows, 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Read the B rows of an fp16 GEMM through a TMA tensor map when they are
// contiguous per tile (no b_row gather): one box load per 64 K instead of one
// bulk copy per row.
bool tma_b(GemmProblem &p, int rows, int bn) {
  p.tma_b = 0;
  if (p.b_row || (reinterpret_cast<uintptr_t>(p.b) & 15) || (p.ldb * 2) % 16) return false;
  if (!make_map(&p.bmap, p.b, rows, p.ldb, p.ldb, bn)) return false;
  p.tma_b = 1;
  return true;
}

// Tensor-core residual GEMM of projection p over the main tile table.
tileq_status tc_args(TcArgs *a, const GemmPlan &g, const LayerInfo &li, const PackedLayout &pl,
                     const void *packed, int p, void *ws, const WsLayout &w, const void *bmat, int bld,
                     int bcols) {
  const ProjInfo &q = li.p[p];
  std::memset(a, 0, sizeof(*a));
  if (!make_map(&a->bmap, bmat, w.plan.P, bcols, bld, g.bn)) return TILEQ_ERR_CUDA;
  a->tiles = at<int4>(ws, g.wide ? w.tiles_wide : w.tiles_main);
  a->tile_count = at<int>(ws, w.tile_counts) + (g.wide ? 1 : 0);
  a->m_tiles = g.m_tiles;
  a->m_rows = g.m_tiles;
  a->ksplit = g.ksplit;
  a->d_out = q.d_out;
  a->d_in = q.d_in;
  a->group = q.group;
  a->n_experts = li.K;
  a->codes[0] = at<uint4>(packed, pl.qw[p]);
  a->sz[0] = at<uint32_t>(packed, pl.sz[p]);
  a->part = at<float>(ws, w.part);
  a->part_items = std::max(g.items, 1);
  a->counters = at<int>(ws, w.counters);
  a->status = at<int>(ws, w.status);
  return TILEQ_OK;
}

// Low-rank K extension of projection slot `slot` (0/1) of a tensor-core GEMM.
void tc_ext(TcArgs *a, int slot, const LayerInfo &li, const PackedLayout &pl, const void *packed, int p,
            int col) {
  const ProjInfo &q = li.p[p];
  a->rank = q.rank;
  a->ext_col[slot] = col;
  a->u[slot] = at<__half>(packed, pl.uf[p]);
  std::memcpy(a->u_blk[slot], q.m_of, kMaxExperts);
}

tileq_status tc_launch(const TcArgs &a, int np, const GemmPlan &g, cudaStream_t stream) {
  return launch_gemm_tc(a, np, g.bn, kNumSMs, stream) == cudaSuccess ? TILEQ_OK : TILEQ_ERR_CUDA;
}

// A dense fp16 product on tcgen05 (gemm_dense.cu): A row-major fp16 (arow[p],
// lda, arows rows; 0 = pad128(d_out)), B the fp16 rows [brows][ldb], items
// either a tile table (of width g.bn) or 0..static_items-1.  np == 2: two
// projections share B (pair units).
struct TcF16 {
  int np = 1;
  const __half *arow[2] = {nullptr, nullptr};
  int lda = 0, d_out = 0, d_in = 0, arows = 0;
  const int4 *tiles = nullptr;
  const int *tile_count = nullptr;
  int static_items = 0;
  const int8_t *a_blk = nullptr;
  const __half *b = nullptr;
  int brows = 0, ldb = 0;
  int epi = EPI_STORE_F32;
  void *out[2] = {nullptr, nullptr};
  int ldo = 0;
  const float *col_scale[2] = {nullptr, nullptr};
  const float *row_scale = nullptr;
};

// Item-tile width of a dense product over `items` items with `m_units` units
// per tile: the fewest CTA waves times the time of one unit, from the measured
// cost of one M=128 K=16 tcgen05.mma (N=64: 48 cycles, N=128: 64, N=256: 128).
int dense_bn(int items, int m_units) {
  int best = 128;
  long long best_cost = -1;
  for (int bn : {256, 128, 64}) {
    const long long units = (long long)cdiv(items, bn) * m_units;
    const long long cost = cdiv(units, kNumSMs) * (bn == 64 ? 48 : bn / 2);
    if (best_cost < 0 || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

tileq_status tc_f16(const TcF16 &f, const GemmPlan &g, void *ws, const WsLayout &w, cudaStream_t stream) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  if (f.d_in % 64 || f.d_in <= 0) return TILEQ_ERR_UNSUPPORTED;
  const int m_blocks = cdiv(f.d_out, 128);
  const bool pair = f.np == 2;
  const int mb = pair || m_blocks > 1 ? 2 : 1;
  a.pair = pair;
  a.m_blocks = m_blocks;
  a.m_units = pair ? m_blocks : cdiv(m_blocks, mb);
  const int bn = f.tiles ? g.bn : dense_bn(f.static_items, a.m_units);
  const int arows = f.arows ? f.arows : m_blocks * 128;
  for (int p = 0; p < f.np; ++p)
    if (!make_map(&a.amap[p], f.arow[p], arows, f.d_in, f.lda, 128)) return TILEQ_ERR_CUDA;
  if (!make_map(&a.bmap, f.b, f.brows, f.ldb, f.ldb, bn)) return TILEQ_ERR_CUDA;
  a.tiles = f.tiles;
  a.tile_count = f.tile_count;
  a.static_items = f.static_items;
  a.use_a_blk = f.a_blk != nullptr;
  if (f.a_blk) std::memcpy(a.a_blk, f.a_blk, kMaxExperts);
  a.d_out = f.d_out;
  a.d_in = f.d_in;
  a.epi = f.epi;
  a.out[0] = f.out[0];
  a.out[1] = f.out[1];
  a.ldo = f.ldo;
  a.col_scale[0] = f.col_scale[0];
  a.col_scale[1] = f.col_scale[1];
  a.row_scale = f.row_scale;
  a.status = at<int>(ws, w.status);
  const long long units = f.tiles ? kNumSMs : (long long)cdiv(f.static_items, bn) * a.m_units;
  const int grid = (int)std::min<long long>(kNumSMs, units);
  return launch_gemm_dense(a, mb, bn, grid, stream) == cudaSuccess ? TILEQ_OK : TILEQ_ERR_CUDA;
}

// One residual projection (or the gate/up pair) over the main tile table:
//   out = epi( s*(q-z) B[:, 0:d_in]  +  U_m B[:, ext .. ext + rank] )
struct Residual {
  int np = 1;
  int proj[2] = {0, 0};
  bool ext = false;
  int ext_col[2] = {0, 0};
  const __half *b = nullptr;
  int ldb = 0;
  int epi = EPI_STORE_F32;
  void *out[2] = {nullptr, nullptr};
  int ldo = 0;
  const float *row_scale = nullptr;
  // decode-regime kernel, one projection: fuse the weighted top-k combine
  // (out_tok = bf16 layer output, yshared = the shared expert or null)
  bool combine = false;
  // decode-regime kernel, gate/up: fp8 mode, B = the e4m3 pieces (ws.x8, per-item
  // scales ws.xs), the extension columns from b
  bool f8 = false;
  int top_k = 0;
  const float *yshared = nullptr;
  void *out_tok = nullptr;
};

tileq_status run_residual_dq(const Residual &r, const GemmPlan &g, const LayerInfo &li, const PackedLayout &pl,
                             const void *packed, void *ws, const WsLayout &w, cudaStream_t stream) {
  DqArgs a;
  std::memset(&a, 0, sizeof(a));
  const ProjInfo &q = li.p[r.proj[0]];
  if (r.f8) {
    a.f8 = 1;
    a.xs = at<float>(ws, w.xs);
    if (!make_map_u8(&a.bmap, at<uint8_t>(ws, w.x8), w.plan.P, 2 * q.d_in, g.bn)) return TILEQ_ERR_CUDA;
    if (!make_map(&a.bmap_ext, r.b, w.plan.P, r.ldb, r.ldb, g.bn)) return TILEQ_ERR_CUDA;
  } else if (!make_map(&a.bmap, r.b, w.plan.P, r.ldb, r.ldb, g.bn)) {
    return TILEQ_ERR_CUDA;
  }
  a.tiles = at<int4>(ws, w.tiles_main);
  a.tile_count = at<int>(ws, w.tile_counts);
  a.max_tiles = g.slots;
  a.m_tiles = g.m_tiles;
  a.d_out = q.d_out;
  a.d_in = q.d_in;
  a.group = q.group;
  a.rank = r.ext ? q.rank : 0;
  for (int i = 0; i < r.np; ++i) {
    const ProjInfo &qi = li.p[r.proj[i]];
    a.codes[i] = at<uint32_t>(packed, pl.qw[r.proj[i]]);
    a.sz[i] = at<uint32_t>(packed, pl.sz[r.proj[i]]);
    if (r.ext) {
      a.ext_col[i] = r.ext_col[i];
      a.u[i] = at<__half>(packed, pl.uf[r.proj[i]]);
      std::memcpy(a.u_blk[i], qi.m_of, kMaxExperts);
    }
  }
  a.epi = r.epi;
  a.out = r.out[0];
  a.out2 = r.out[1];
  a.ldo = r.ldo;
  a.row_scale = r.row_scale;
  a.part = at<float>(ws, w.part);
  a.counters = at<int>(ws, w.counters);
  a.status = at<int>(ws, w.status);
  if (r.combine) {
    a.combine = 1;
    a.top_k = r.top_k;
    a.slot_tok = at<int>(ws, w.slot_tok);
    a.slot_of_pair = at<int>(ws, w.slot_of_pair);
    a.yshared = r.yshared;
    a.out_tok = static_cast<__nv_bfloat16 *>(r.out_tok);
    a.tok_counters = at<int>(ws, w.tokcnt);
  }
  return launch_gemm_dq(a, r.np, g.bn, stream) == cudaSuccess ? TILEQ_OK : TILEQ_ERR_CUDA;
}

tileq_status run_residual(const Residual &r, const GemmPlan &g, const LayerInfo &li, const PackedLayout &pl,
                          const void *packed, void *ws, const WsLayout &w, cudaStream_t stream) {
  if (g.dq) return run_residual_dq(r, g, li, pl, packed, ws, w, stream);
  TcArgs a;
  tileq_status st = tc_args(&a, g, li, pl, packed, r.proj[0], ws, w, r.b, r.ldb, r.ldb);
  if (st != TILEQ_OK) return st;
  for (int i = 0; i < r.np; ++i) {
    // tcgen05 reads the row layout of the codes, warp MMA the fragment layout
    a.codes[i] = at<uint4>(packed, g.tc ? pl.qw[r.proj[i]] : pl.qf[r.proj[i]]);
    const bool q3 = li.p[r.proj[i]].bits == 3;
    a.codes_hi[i] = q3 && !g.tc ? at<uint2>(packed, pl.qfh[r.proj[i]]) : nullptr;
    a.codes_hi_rows[i] = q3 && g.tc ? at<uint32_t>(packed, pl.qwh[r.proj[i]]) : nullptr;
    a.sz[i] = at<uint32_t>(packed, pl.sz[r.proj[i]]);
    if (r.ext) tc_ext(&a, i, li, pl, packed, r.proj[i], r.ext_col[i]);
  }
  a.epi = r.epi;
  a.out[0] = r.out[0];
  a.out[1] = r.out[1];
  a.ldo = r.ldo;
  a.row_scale = r.row_scale;
  if (g.row_pair) {
    // both halves of the pair read projection r.proj[0]
    a.row_pair = 1;
    a.m_rows = cdiv(li.p[r.proj[0]].d_out, 128);
    a.codes[1] = a.codes[0];
    a.codes_hi_rows[1] = a.codes_hi_rows[0];
    a.sz[1] = a.sz[0];
    a.u[1] = a.u[0];
    a.ext_col[1] = a.ext_col[0];
    std::memcpy(a.u_blk[1], a.u_blk[0], kMaxExperts);
    return tc_launch(a, 2, g, stream);
  }
  if (g.tc) return tc_launch(a, r.np, g, stream);
  return launch_gemm_q2(a, r.np, g.bn, g.slots, stream) == cudaSuccess ? TILEQ_OK : TILEQ_ERR_CUDA;
}

tileq_status run_route_permute(const tileq_layer *L, const LayerInfo &li, const WsLayout &w,
                               const void *x, int T, const float *logits, int top_k, void *ws,
                               int n_zproj, const int zproj_ids[2], int row_proj,
                               cudaStream_t stream) {
  RouteArgs ra;
  ra.logits = logits;
  ra.x = static_cast<const __nv_bfloat16 *>(x);
  ra.x16 = at<__half>(ws, w.x16);
  ra.d_x = li.d_x;
  ra.T = T;
  ra.K = L->K;
  ra.k = top_k;
  ra.full_softmax = L->route_mode == TILEQ_ROUTE_FULL_SOFTMAX;
  ra.topk_idx = at<int32_t>(ws, w.topk_idx);
  ra.topk_w = at<float>(ws, w.topk_w);
  ra.zero = at<int>(ws, w.counters);
  ra.nzero = w.n_counters;
  ra.status = at<int>(ws, w.status);
  mark(ST_BEGIN, stream);
  const long long xchunks = x ? (long long)T * li.d_x / 8 : 0;
  const int P = T * top_k;

  PermuteArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  pa.T = T;
  pa.k = top_k;
  pa.K = L->K;
  pa.M = L->M;
  pa.N = L->N;
  pa.bn = w.plan.bn_main;
  pa.topk_idx = ra.topk_idx;
  pa.topk_w = ra.topk_w;
  pa.dest = at<int>(ws, w.dest);
  pa.expert_offsets = at<int32_t>(ws, w.expert_offsets);
  pa.sorted_pairs = at<int32_t>(ws, w.sorted_pairs);
  pa.slot_of_pair = at<int>(ws, w.slot_of_pair);
  pa.slot_tok = at<int>(ws, w.slot_tok);
  pa.slot_w = at<float>(ws, w.slot_w);
  pa.tiles_main = at<int4>(ws, w.tiles_main);
  pa.tile_first_main = at<int>(ws, w.tile_first);
  pa.tile_counts = at<int>(ws, w.tile_counts);
  pa.bn_wide = w.plan.bn_wide;
  pa.tiles_wide = at<int4>(ws, w.tiles_wide);
  pa.n_zproj = n_zproj;
  for (int z = 0; z < 2; ++z) {
    if (z < n_zproj) std::memcpy(pa.n_of[z], li.p[zproj_ids[z]].n_of, kMaxExperts);
    pa.zidx[z] = at<int>(ws, w.zidx[z]);
  }
  pa.row_proj = row_proj;
  if (row_proj >= 0) std::memcpy(pa.m_of_row, li.p[row_proj].m_of, kMaxExperts);
  pa.aidx = at<int>(ws, w.aidx);
  pa.pcounts = at<int>(ws, w.pcounts);
  if (P <= kPermMultiMin) {
    // one launch: CTA 0 routes and sorts, the others zero the counters and
    // convert x (at most four 16-byte chunks per thread of 1024-thread CTAs)
    const unsigned cblocks = std::min(std::max(nblocks(xchunks, 1024 * 4), nblocks(w.n_counters, 1024)),
                                      (unsigned)(2 * kNumSMs));
    TQ_CUDA(launch_pdl(route_permute_kernel, dim3(1 + cblocks), dim3(1024), 0, stream, ra, pa));
    TQ_LAUNCHED();
    mark(ST_ROUTE, stream);
    mark(ST_PERMUTE, stream);
    return TILEQ_OK;
  }
  // one warp per token for the top-k; enough blocks that the x conversion has
  // at most four 16-byte chunks per thread
  const unsigned rblocks = std::max(nblocks(T, 8), std::min(nblocks(xchunks, 256 * 4), (unsigned)(8 * kNumSMs)));
  TQ_CUDA(launch_pdl(route_kernel, dim3(rblocks), dim3(256), 0, stream, ra));
  TQ_LAUNCHED();
  mark(ST_ROUTE, stream);
  {
    const unsigned nc = (unsigned)cdiv(P, kPermChunk);
    TQ_CUDA(launch_pdl(permute_count_kernel, dim3(nc), dim3(kPermChunkThreads), 0, stream, pa));
    TQ_LAUNCHED();
    TQ_CUDA(launch_pdl(permute_scatter_kernel, dim3(nc), dim3(kPermChunkThreads), 0, stream, pa));
    TQ_LAUNCHED();
  }
  mark(ST_PERMUTE, stream);
  return TILEQ_OK;
}

tileq_status copy_route_out(const tileq_layer *L, const WsLayout &w, void *ws, int T, int top_k,
                            tileq_route_out *route, cudaStream_t stream) {
  if (!route) return TILEQ_OK;
  const size_t P = (size_t)T * top_k;
  if (route->topk_idx)
    TQ_CUDA(cudaMemcpyAsync(route->topk_idx, at<int32_t>(ws, w.topk_idx), P * 4,
                            cudaMemcpyDeviceToDevice, stream));
  if (route->topk_w)
    TQ_CUDA(cudaMemcpyAsync(route->topk_w, at<float>(ws, w.topk_w), P * 4,
                            cudaMemcpyDeviceToDevice, stream));
  if (route->expert_offsets)
    TQ_CUDA(cudaMemcpyAsync(route->expert_offsets, at<int32_t>(ws, w.expert_offsets),
                            (L->K + 1) * 4, cudaMemcpyDeviceToDevice, stream));
  if (route->sorted_pairs)
    TQ_CUDA(cudaMemcpyAsync(route->sorted_pairs, at<int32_t>(ws, w.sorted_pairs), P * 4,
                            cudaMemcpyDeviceToDevice, stream));
  return TILEQ_OK;
}

// The always-on shared expert (dense fp16 SwiGLU) into the fp32 buffer ys;
// *yshared = ys, or null without a shared expert.
// A side stream per host thread and device, with its fork and join events,
// for work of a forward that does not depend on the routing (the shared
// expert).  Created on first use; if that fails the work stays on the
// caller's stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool tried = false, ok = false;
};
SideStream &side_stream() {
  constexpr int kDevices = 64;
  static thread_local SideStream per_device[kDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) {
    cudaGetLastError();
    static thread_local SideStream none;
    none.tried = true;
    return none;
  }
  SideStream &sd = per_device[dev];
  if (!sd.tried) {
    sd.tried = true;
    sd.ok = cudaStreamCreateWithFlags(&sd.s, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming) == cudaSuccess;
    if (!sd.ok) cudaGetLastError();
  }
  return sd;
}

tileq_status run_shared(const tileq_layer *L, const PackedLayout &pl, const WsLayout &w, const void *packed,
                        void *ws, int T, const float **yshared_out, cudaStream_t stream) {
  const float *yshared = nullptr;
  if (L->shared_d_ff > 0 && w.plan.sh_gu.tc) {
    const int Fs = L->shared_d_ff, D = L->d_model;
    TcF16 f;
    f.np = 2;
    f.arow[0] = at<__half>(packed, pl.shr[0]);
    f.arow[1] = at<__half>(packed, pl.shr[1]);
    f.lda = D;
    f.d_out = Fs;
    f.d_in = D;
    f.static_items = T;
    f.b = at<__half>(ws, w.x16);
    f.brows = T;
    f.ldb = D;
    f.epi = EPI_SWIGLU_H;
    f.out[0] = at<__half>(ws, w.hs);
    f.ldo = Fs;
    if (tc_f16(f, w.plan.sh_gu, ws, w, stream) != TILEQ_OK) return TILEQ_ERR_CUDA;
    TcF16 d;
    d.arow[0] = at<__half>(packed, pl.shr[2]);
    d.lda = Fs;
    d.d_out = D;
    d.d_in = Fs;
    d.static_items = T;
    d.b = at<__half>(ws, w.hs);
    d.brows = T;
    d.ldb = Fs;
    d.epi = EPI_STORE_F32;
    d.out[0] = at<float>(ws, w.ys);
    d.ldo = D;
    if (tc_f16(d, w.plan.sh_down, ws, w, stream) != TILEQ_OK) return TILEQ_ERR_CUDA;
    yshared = at<float>(ws, w.ys);
  } else if (L->shared_d_ff > 0) {
    const int Fs = L->shared_d_ff, D = L->d_model;
    GemmBatch b;
    b.p[0] = problem(w.plan.sh_gu, ws, w);
    GemmProblem &g = b.p[0];
    g.static_items = T;
    g.d_out = Fs;
    g.d_in = D;
    g.a[0] = at<uint4>(packed, pl.sh[0]);
    g.a[1] = at<uint4>(packed, pl.sh[1]);
    g.b = at<__half>(ws, w.x16);
    g.ldb = D;
    g.epi = EPI_SWIGLU_H;
    g.out[0] = at<__half>(ws, w.hs);
    g.ldo = Fs;
    tma_b(g, T, w.plan.sh_gu.bn);
    if (gemm(b, 1, 2, w.plan.sh_gu, stream) != TILEQ_OK) return TILEQ_ERR_CUDA;
    b.p[0] = problem(w.plan.sh_down, ws, w);
    GemmProblem &d = b.p[0];
    d.static_items = T;
    d.d_out = D;
    d.d_in = Fs;
    d.a[0] = at<uint4>(packed, pl.sh[2]);
    d.b = at<__half>(ws, w.hs);
    d.ldb = Fs;
    d.epi = EPI_STORE_F32;
    d.out[0] = at<float>(ws, w.ys);
    d.ldo = D;
    tma_b(d, T, w.plan.sh_down.bn);
    if (gemm(b, 1, 1, w.plan.sh_down, stream) != TILEQ_OK) return TILEQ_ERR_CUDA;
    yshared = at<float>(ws, w.ys);
  }
  *yshared_out = yshared;
  return TILEQ_OK;
}

// The weighted top-k combine / unpermute of the per-slot outputs (the slot
// weights are already applied), plus the shared expert.
tileq_status run_combine(const LayerInfo &li, const WsLayout &w, void *ws, int T, int top_k, const float *yshared,
                         void *out, cudaStream_t stream) {
  CombineArgs ca;
  ca.T = T;
  ca.k = top_k;
  ca.d = li.d_y;
  ca.slot_of_pair = at<int>(ws, w.slot_of_pair);
  ca.ybuf = at<float>(ws, w.ybuf);
  ca.yshared = yshared;
  ca.out = static_cast<__nv_bfloat16 *>(out);
  if (launch_combine(ca, stream) != cudaSuccess) return TILEQ_ERR_CUDA;
  count_launches();
  return TILEQ_OK;
}

tileq_status check_forward_args(const tileq_layer *layer, LayerInfo *li, const void *packed,
                                const void *x, int T, const float *logits, int top_k, void *out,
                                void *ws, size_t ws_bytes) {
  tileq_status st = validate_layer(layer, li);
  if (st != TILEQ_OK) return st;
  if (T < 0 || top_k < 1 || top_k > layer->K || top_k > kMaxTopK) return TILEQ_ERR_INVALID_ARG;
  if (T == 0) return TILEQ_OK;
  if (!packed || !x || !logits || !out || !ws) return TILEQ_ERR_INVALID_ARG;
  if ((long long)T * top_k > (1LL << 24)) return TILEQ_ERR_UNSUPPORTED;
  const WsLayout w = ws_layout(layer, *li, T, top_k);
  if (ws_bytes < w.total) return TILEQ_ERR_WORKSPACE;
  return TILEQ_OK;
}

LrAccArgs lracc_args(const ProjInfo &q, const WsLayout &w, void *ws, int top_k, __half *out, int ld,
                     int col) {
  LrAccArgs la;
  std::memset(&la, 0, sizeof(la));
  la.P = w.plan.P;
  la.k = top_k;
  la.r = q.rank;
  la.sorted_pairs = at<int32_t>(ws, w.sorted_pairs);
  la.aidx = at<int>(ws, w.aidx);
  la.topk_idx = at<int32_t>(ws, w.topk_idx);
  la.topk_w = at<float>(ws, w.topk_w);
  std::memcpy(la.m_of, q.m_of, kMaxExperts);
  la.slot_of_pair = at<int>(ws, w.slot_of_pair);
  la.out = out;
  la.ld = ld;
  la.col = col;
  la.status = at<int>(ws, w.status);
  return la;
}

// z_{t,n} = Sigma * (V_n^T x_t) once per distinct (token, grid column): one
// grouped GEMM per projection (gate and up share a launch).
tileq_status run_zproj(const tileq_layer *layer, const LayerInfo &li, const PackedLayout &pl,
                       const void *packed, const WsLayout &w, void *ws, int nz,
                       cudaStream_t stream) {
  if (w.plan.zproj.tc) {
    // all projections of the launch in one tcgen05 pass (gate and up share B = x)
    const ProjInfo &q = li.p[0];
    TcF16 f;
    f.np = nz;
    for (int p = 0; p < nz; ++p) {
      f.arow[p] = at<__half>(packed, pl.vr[p]);
      f.out[p] = at<float>(ws, w.zc[p]);
      f.col_scale[p] = at<float>(packed, pl.sig[p]);
    }
    f.lda = q.d_in;
    f.d_out = layer->N * pad128(q.rank);
    f.d_in = q.d_in;
    f.static_items = w.plan.T;
    f.b = at<__half>(ws, w.x16);
    f.brows = w.plan.T;
    f.ldb = q.d_in;
    f.epi = nz == 2 ? EPI_STORE2_F32 : EPI_STORE_F32;
    f.ldo = f.d_out;
    return tc_f16(f, w.plan.zproj, ws, w, stream);
  }
  GemmBatch b;
  for (int p = 0; p < nz; ++p) {
    const ProjInfo &q = li.p[p];
    b.p[p] = problem(w.plan.zproj, ws, w);
    GemmProblem &z = b.p[p];
    z.static_items = w.plan.T;
    z.d_out = layer->N * pad128(q.rank);
    z.d_in = q.d_in;
    z.a[0] = at<uint4>(packed, pl.vf[p]);
    z.b = at<__half>(ws, w.x16);
    z.ldb = q.d_in;
    z.epi = EPI_PARTIAL_F32;
    z.col_scale = at<float>(packed, pl.sig[p]);
    z.out[0] = at<float>(ws, w.zc[p]);
    z.ldo = z.d_out;
    tma_b(z, w.plan.T, w.plan.zproj.bn);
    z.part = at<float>(ws, w.part) + (size_t)p * w.part_zstride;
  }
  return gemm(b, nz, 1, w.plan.zproj, stream);
}

}  // namespace

extern "C" {

const char *tileq_status_string(tileq_status s) {
  switch (s) {
    case TILEQ_OK: return "TILEQ_OK";
    case TILEQ_ERR_INVALID_ARG: return "TILEQ_ERR_INVALID_ARG";
    case TILEQ_ERR_UNSUPPORTED: return "TILEQ_ERR_UNSUPPORTED";
    case TILEQ_ERR_WORKSPACE: return "TILEQ_ERR_WORKSPACE";
    case TILEQ_ERR_CUDA: return "TILEQ_ERR_CUDA";
    case TILEQ_ERR_TIMEOUT: return "TILEQ_ERR_TIMEOUT";
    case TILEQ_ERR_RANGE: return "TILEQ_ERR_RANGE";
  }
  return "TILEQ_UNKNOWN_STATUS";
}

tileq_status tileq_packed_size(const tileq_layer *layer, size_t *bytes) {
  LayerInfo li;
  if (!bytes) return TILEQ_ERR_INVALID_ARG;
  tileq_status st = validate_layer(layer, &li, false);
  if (st != TILEQ_OK) return st;
  *bytes = packed_layout(layer, li).total;
  return TILEQ_OK;
}

tileq_status tileq_pack(const tileq_layer *layer, void *packed, size_t packed_bytes,
                        tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  LayerInfo li;
  tileq_status st = validate_layer(layer, &li);
  if (st != TILEQ_OK) return st;
  if (!packed) return TILEQ_ERR_INVALID_ARG;
  const PackedLayout pl = packed_layout(layer, li);
  if (packed_bytes < pl.total) return TILEQ_ERR_WORKSPACE;
  const int K = layer->K;
  for (int p = 0; p < li.nproj; ++p) {
    const tileq_proj &src = layer->proj[p];
    const ProjInfo &q = li.p[p];
    {
      const long long n = (long long)K * (pad128(q.d_out) / 128) * (q.d_in / 128) * 128 * 8;
      pack_codes_tc_kernel<<<nblocks(n, 256), 256, 0, stream>>>(src.codes, at<uint32_t>(packed, pl.qw[p]),
                                                                 K, q.d_out, q.d_in);
      TQ_LAUNCHED();
      pack_codes_kernel<<<nblocks(n / 4, 256), 256, 0, stream>>>(src.codes, at<uint4>(packed, pl.qf[p]),
                                                                 K, q.d_out, q.d_in);
      TQ_LAUNCHED();
      if (q.bits == 3) {
        pack_codes_hi_kernel<<<nblocks(n / 4, 256), 256, 0, stream>>>(src.codes_hi, at<uint2>(packed, pl.qfh[p]),
                                                                      K, q.d_out, q.d_in);
        TQ_LAUNCHED();
        pack_codes_tc_hi_kernel<<<nblocks(n / 2, 256), 256, 0, stream>>>(
            src.codes_hi, at<uint32_t>(packed, pl.qwh[p]), K, q.d_out, q.d_in);
        TQ_LAUNCHED();
      }
    }
    {
      const long long n = (long long)K * pad128(q.d_out) * q.G;
      pack_sz_kernel<<<nblocks(n, 256), 256, 0, stream>>>(static_cast<const __half *>(src.scales),
                                                           src.zeros, at<uint32_t>(packed, pl.sz[p]),
                                                           K, q.d_out, q.G, q.bits);
      TQ_LAUNCHED();
    }
    if (q.rank > 0) {
      const __nv_bfloat16 *U = static_cast<const __nv_bfloat16 *>(src.U);
      const __nv_bfloat16 *V = static_cast<const __nv_bfloat16 *>(src.V);
      // U block m: fp16 rows (padded to 128), the K extension of the residual GEMM
      long long n = (long long)layer->M * pad128(q.d_out) * q.rank;
      pack_rows_f16_kernel<<<nblocks(n, 256), 256, 0, stream>>>(U, layer->M, q.d_out, q.rank,
                                                                 at<__half>(packed, pl.uf[p]));
      TQ_LAUNCHED();
      // V_n^T: rows i (rank), cols k (d_in): element at V[(n*d_in + k)*rank + i]
      n = (long long)frag_bytes(layer->N, q.rank, q.d_in, 8) / 16;
      pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(V, (long long)q.d_in * q.rank, 1, q.rank,
                                                             layer->N, q.rank, q.d_in, 8,
                                                             at<uint4>(packed, pl.vf[p]));
      TQ_LAUNCHED();
      const int ns = layer->N * pad128(q.rank);
      expand_sigma_kernel<<<nblocks(ns, 256), 256, 0, stream>>>(src.Sigma, q.rank, pad128(q.rank), layer->N,
                                                                at<float>(packed, pl.sig[p]));
      TQ_LAUNCHED();
      n = (long long)layer->N * pad128(q.rank) * q.d_in;
      pack_vt_rows_kernel<<<nblocks(n, 256), 256, 0, stream>>>(V, layer->N, q.rank, q.d_in,
                                                                 at<__half>(packed, pl.vr[p]));
      TQ_LAUNCHED();
    }
  }
  if (layer->shared_d_ff > 0) {
    const int Fs = layer->shared_d_ff, D = layer->d_model;
    for (int i = 0; i < 3; ++i) {
      const int R = i < 2 ? Fs : D, Cc = i < 2 ? D : Fs;
      const long long n = (long long)frag_bytes(1, R, Cc, 8) / 16;
      pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16 *>(layer->shared_w[i]), 0, Cc, 1, 1, R, Cc, 8,
          at<uint4>(packed, pl.sh[i]));
      TQ_LAUNCHED();
      const long long nr = (long long)pad128(R) * Cc;
      pack_rows_f16_kernel<<<nblocks(nr, 256), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16 *>(layer->shared_w[i]), 1, R, Cc, at<__half>(packed, pl.shr[i]));
      TQ_LAUNCHED();
    }
  }
  return TILEQ_OK;
}

tileq_status tileq_workspace_size(const tileq_layer *layer, int T, int top_k, size_t *bytes) {
  LayerInfo li;
  if (!bytes) return TILEQ_ERR_INVALID_ARG;
  tileq_status st = validate_layer(layer, &li, false);
  if (st != TILEQ_OK) return st;
  if (T < 0 || top_k < 1 || top_k > layer->K || top_k > kMaxTopK) return TILEQ_ERR_INVALID_ARG;
  *bytes = ws_layout(layer, li, T, top_k).total;
  return TILEQ_OK;
}

tileq_status tileq_moe_forward(const tileq_layer *layer, const void *packed, const void *x, int T,
                               const float *router_logits, int top_k, void *out, void *ws,
                               size_t ws_bytes, tileq_route_out *route, tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  LayerInfo li;
  tileq_status st = check_forward_args(layer, &li, packed, x, T, router_logits, top_k, out, ws, ws_bytes);
  if (st != TILEQ_OK || T == 0) return st;
  const PackedLayout pl = packed_layout(layer, li);
  const WsLayout w = ws_layout(layer, li, T, top_k);
  const Plan &plan = w.plan;
  __half *xext = at<__half>(ws, w.xext);

  if (layer->kind == TILEQ_LINEAR) {
    const ProjInfo &q = li.p[0];
    const int zids[2] = {0, 0};
    st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, q.rank > 0 ? 1 : 0, zids,
                           q.rank > 0 ? 0 : -1, stream);
    if (st != TILEQ_OK) return st;
    // x' = w * x per slot in the first d_in columns of the activation matrix
    ScaleGatherArgs sg{plan.P, q.d_in, w.ld_x, at<int>(ws, w.slot_tok), at<float>(ws, w.slot_w),
                       at<__half>(ws, w.x16), xext};
    TQ_CUDA(launch_pdl(scale_gather_kernel, dim3(nblocks((long long)plan.P * (q.d_in / 2), 256)), dim3(256), 0, stream, sg));
    TQ_LAUNCHED();
    if (q.rank > 0) {
      if ((st = run_zproj(layer, li, pl, packed, w, ws, 1, stream)) != TILEQ_OK) return st;
      mark(ST_ZPROJ, stream);
      mark(ST_GATEUP, stream);
      // a_{t,m} = sum_j w_j z_{t,n_j} over the token's experts in grid row m -> columns d_in..
      LrAccArgs la = lracc_args(q, w, ws, top_k, xext, w.ld_x, q.d_in);
      la.zcol = at<float>(ws, w.zc[0]);
      la.zidx = at<int>(ws, w.zidx[0]);
      la.zld = pad128(q.rank);
      la.zks = plan.zproj.ksplit;
      la.zsplit = (long long)T * layer->N * pad128(q.rank);
      TQ_CUDA(launch_pdl(lr_accumulate_kernel, dim3(nblocks((long long)plan.P * 32, 256)), dim3(256), 0, stream, la));
      TQ_LAUNCHED();
      mark(ST_ZDOWN, stream);
    } else {
      mark(ST_ZPROJ, stream);
      mark(ST_GATEUP, stream);
      mark(ST_ZDOWN, stream);
    }
    mark(ST_SHARED, stream);
    Residual r;
    r.ext = q.rank > 0;
    r.ext_col[0] = q.d_in;
    r.b = xext;
    r.ldb = w.ld_x;
    r.out[0] = at<float>(ws, w.ybuf);
    r.ldo = q.d_out;
    r.combine = plan.linear.dq;
    r.top_k = top_k;
    r.out_tok = out;
    if ((st = run_residual(r, plan.linear, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    mark(ST_RESIDUAL, stream);
    if (!r.combine && (st = run_combine(li, w, ws, T, top_k, nullptr, out, stream)) != TILEQ_OK) return st;
    mark(ST_COMBINE, stream);
  } else {
    const ProjInfo &qg = li.p[0], &qd = li.p[2];
    const int zids[2] = {0, 1};
    const bool lr_gu = qg.rank > 0, lr_d = qd.rank > 0;
    st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, lr_gu ? 2 : 0, zids, -1, stream);
    if (st != TILEQ_OK) return st;
    const int D = layer->d_model, F = layer->d_ff;
    __half *hext = at<__half>(ws, w.hext);
    // the shared expert reads x alone: it runs on the side stream from here,
    // beside the routed GEMMs, with its own split-K regions
    const float *yshared = nullptr;
    SideStream *side = nullptr;
    if (layer->shared_d_ff > 0) {
      SideStream &sd = side_stream();
      if (sd.ok) {
        WsLayout wsh = w;
        wsh.part = w.part_sh;
        wsh.counters = w.counters_sh;
        TQ_CUDA(cudaEventRecord(sd.fork, stream));
        TQ_CUDA(cudaStreamWaitEvent(sd.s, sd.fork, 0));
        if ((st = run_shared(layer, pl, wsh, packed, ws, T, &yshared, sd.s)) != TILEQ_OK) return st;
        TQ_CUDA(cudaEventRecord(sd.join, sd.s));
        side = &sd;
      }
    }
    if (lr_gu && (st = run_zproj(layer, li, pl, packed, w, ws, 2, stream)) != TILEQ_OK) return st;
    {
      // activation matrix of gate/up: [x_t | z^gate_{t,n} | z^up_{t,n}] per slot
      GatherExtArgs ga;
      ga.P = plan.P;
      ga.d = D;
      ga.r = qg.rank;
      ga.ld = w.ld_x;
      ga.slot_tok = at<int>(ws, w.slot_tok);
      ga.x16 = at<__half>(ws, w.x16);
      ga.z[0] = lr_gu ? at<float>(ws, w.zc[0]) : nullptr;
      ga.z[1] = lr_gu ? at<float>(ws, w.zc[1]) : nullptr;
      ga.zks = plan.zproj.ksplit;
      ga.zsplit = (long long)T * layer->N * pad128(qg.rank);
      ga.zidx[0] = at<int>(ws, w.zidx[0]);
      ga.zidx[1] = at<int>(ws, w.zidx[1]);
      ga.zld = pad128(qg.rank);
      ga.out = xext;
      ga.T = T;
      ga.k = top_k;
      ga.slot_of_pair = at<int>(ws, w.slot_of_pair);
      ga.status = at<int>(ws, w.status);
      if (plan.gateup.dq) {
        // fp8 decode GEMM: e4m3 pieces of each slot's x (and its z columns, scaled alike)
        GatherX8Args g8;
        std::memset(&g8, 0, sizeof(g8));
        g8.T = T;
        g8.k = top_k;
        g8.d = D;
        g8.r = qg.rank;
        g8.ld = w.ld_x;
        g8.slot_of_pair = ga.slot_of_pair;
        g8.x16 = ga.x16;
        g8.x8 = at<uint8_t>(ws, w.x8);
        g8.xs = at<float>(ws, w.xs);
        g8.z[0] = ga.z[0];
        g8.z[1] = ga.z[1];
        g8.zidx[0] = ga.zidx[0];
        g8.zidx[1] = ga.zidx[1];
        g8.zld = ga.zld;
        g8.zks = ga.zks;
        g8.zsplit = ga.zsplit;
        g8.xext = xext;
        g8.status = ga.status;
        TQ_CUDA(launch_pdl(gather_x8_kernel, dim3(T), dim3(256), 0, stream, g8));
        TQ_LAUNCHED();
      } else {
        const long long chunks = (long long)T * (D / 8) + (long long)plan.P * (lr_gu ? 2 * qg.rank / 8 : 0);
        TQ_CUDA(launch_pdl(gather_ext_kernel, dim3(gather_blocks(chunks)), dim3(256), 0, stream, ga));
        TQ_LAUNCHED();
      }
    }
    mark(ST_ZPROJ, stream);
    {
      // gate/up residual + U_m z (K extension) + SwiGLU; h = w * silu(g) * u per slot
      Residual r;
      r.np = 2;
      r.proj[1] = 1;
      r.ext = lr_gu;
      r.ext_col[0] = D;
      r.ext_col[1] = D + qg.rank;
      r.b = xext;
      r.ldb = w.ld_x;
      r.epi = EPI_SWIGLU_H;
      r.out[0] = hext;
      r.ldo = w.ld_h;
      r.row_scale = at<float>(ws, w.slot_w);
      r.f8 = plan.gateup.dq;
      if ((st = run_residual(r, plan.gateup, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    }
    mark(ST_GATEUP, stream);
    if (lr_d) {
      // z'_slot = Sigma * (V_n^T h_slot) in fp16 into the K-extension columns
      // F .. F + r of the slot's row of h: the down GEMM then adds U_m z'_slot
      // per slot, and the combine's sum over the token's slots carries out the
      // accumulation per grid row (TileQ paper, section 2.2, the in-place
      // accumulation buffer), with the routing weight already inside h
      if (plan.zdown.tc) {
        TcF16 f;
        f.arow[0] = at<__half>(packed, pl.vr[2]);
        f.lda = F;
        f.arows = layer->N * pad128(qd.rank);
        f.d_out = qd.rank;
        f.d_in = F;
        f.tiles = at<int4>(ws, w.tiles_main);
        f.tile_count = at<int>(ws, w.tile_counts);
        f.a_blk = qd.n_of;
        f.b = hext;
        f.brows = plan.P;
        f.ldb = w.ld_h;
        f.epi = EPI_STORE_F16;
        f.out[0] = hext + F;
        f.ldo = w.ld_h;
        f.col_scale[0] = layer->proj[2].Sigma;
        if ((st = tc_f16(f, plan.zdown, ws, w, stream)) != TILEQ_OK) return st;
      } else {
      GemmBatch b;
      b.p[0] = problem(plan.zdown, ws, w);
      GemmProblem &z = b.p[0];
      z.tiles = at<int4>(ws, w.tiles_main);
      z.tile_count = at<int>(ws, w.tile_counts);
      z.d_out = qd.rank;
      z.d_in = F;
      z.a[0] = at<uint4>(packed, pl.vf[2]);
      z.use_a_blk = 1;
      std::memcpy(z.a_blk, qd.n_of, kMaxExperts);
      z.b = hext;
      z.ldb = w.ld_h;
      z.epi = EPI_STORE_F16;
      z.col_scale = layer->proj[2].Sigma;
      z.out[0] = hext + F;
      z.ldo = w.ld_h;
      tma_b(z, plan.P, plan.zdown.bn);
      if ((st = gemm(b, 1, 1, plan.zdown, stream)) != TILEQ_OK) return st;
      }
      mark(ST_ZDOWN, stream);
    } else {
      mark(ST_ZDOWN, stream);
    }
    if (!side) {
      WsLayout wsh = w;
      wsh.part = w.part_sh;
      wsh.counters = w.counters_sh;
      if ((st = run_shared(layer, pl, wsh, packed, ws, T, &yshared, stream)) != TILEQ_OK) return st;
    }
    mark(ST_SHARED, stream);
    Residual r;
    r.proj[0] = 2;
    r.ext = lr_d;
    r.ext_col[0] = F;
    r.b = hext;
    r.ldb = w.ld_h;
    r.out[0] = at<float>(ws, w.ybuf);
    r.ldo = D;
    r.combine = plan.down.dq;
    r.top_k = top_k;
    r.yshared = yshared;
    r.out_tok = out;
    // join the shared expert before its first reader: the combine (fused into
    // the tcgen05 decode down GEMM, or its own kernel)
    if (side && r.combine) TQ_CUDA(cudaStreamWaitEvent(stream, side->join, 0));
    if ((st = run_residual(r, plan.down, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    mark(ST_RESIDUAL, stream);
    if (side && !r.combine) TQ_CUDA(cudaStreamWaitEvent(stream, side->join, 0));
    if (!r.combine && (st = run_combine(li, w, ws, T, top_k, yshared, out, stream)) != TILEQ_OK) return st;
    mark(ST_COMBINE, stream);
  }
  return copy_route_out(layer, w, ws, T, top_k, route, stream);
}

tileq_status tileq_packed_per_expert_size(const tileq_layer *layer, size_t *bytes) {
  LayerInfo li;
  if (!bytes) return TILEQ_ERR_INVALID_ARG;
  tileq_status st = validate_layer(layer, &li, false);
  if (st != TILEQ_OK) return st;
  *bytes = pe_layout(layer, li).total;
  return TILEQ_OK;
}

tileq_status tileq_pack_per_expert(const tileq_layer *layer, const tileq_per_expert_lr *pe,
                                   void *packed_pe, size_t packed_pe_bytes, tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  LayerInfo li;
  tileq_status st = validate_layer(layer, &li, false);
  if (st != TILEQ_OK) return st;
  if (!pe || !packed_pe) return TILEQ_ERR_INVALID_ARG;
  const PePackedLayout pl = pe_layout(layer, li);
  if (packed_pe_bytes < pl.total) return TILEQ_ERR_WORKSPACE;
  const int K = layer->K;
  for (int p = 0; p < li.nproj; ++p) {
    const ProjInfo &q = li.p[p];
    if (q.rank == 0) continue;
    if (!pe->U_pe[p] || !pe->V_pe[p]) return TILEQ_ERR_INVALID_ARG;
    long long n = (long long)frag_bytes(K, q.d_out, q.rank, 8) / 16;
    pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(pe->U_pe[p]), (long long)q.d_out * q.rank, q.rank, 1, K,
        q.d_out, q.rank, 8, at<uint4>(packed_pe, pl.uf[p]));
    TQ_LAUNCHED();
    n = (long long)frag_bytes(K, q.rank, q.d_in, 8) / 16;
    pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(pe->V_pe[p]), (long long)q.d_in * q.rank, 1, q.rank, K,
        q.rank, q.d_in, 8, at<uint4>(packed_pe, pl.vf[p]));
    TQ_LAUNCHED();
    n = (long long)K * pad128(q.d_out) * q.rank;
    pack_rows_f16_kernel<<<nblocks(n, 256), 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(pe->U_pe[p]), K,
                                                               q.d_out, q.rank, at<__half>(packed_pe, pl.ur[p]));
    TQ_LAUNCHED();
    n = (long long)K * pad128(q.rank) * q.d_in;
    pack_vt_rows_kernel<<<nblocks(n, 256), 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(pe->V_pe[p]), K,
                                                               q.rank, q.d_in, at<__half>(packed_pe, pl.vr[p]));
    TQ_LAUNCHED();
  }
  return TILEQ_OK;
}

tileq_status tileq_moe_forward_unfused(const tileq_layer *layer, const void *packed,
                                       const void *packed_pe, const void *x, int T,
                                       const float *router_logits, int top_k, void *out, void *ws,
                                       size_t ws_bytes, tileq_route_out *route,
                                       tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  LayerInfo li;
  tileq_status st = check_forward_args(layer, &li, packed, x, T, router_logits, top_k, out, ws, ws_bytes);
  if (st != TILEQ_OK || T == 0) return st;
  if (!packed_pe) return TILEQ_ERR_INVALID_ARG;
  const PackedLayout pl = packed_layout(layer, li);
  const PePackedLayout ppl = pe_layout(layer, li);
  const WsLayout w = ws_layout(layer, li, T, top_k);
  const Plan &plan = w.plan;
  const int K = layer->K;
  const int zids[2] = {0, 0};
  __half *xext = at<__half>(ws, w.xext);
  st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, 0, zids, -1, stream);
  if (st != TILEQ_OK) return st;

  // Per-expert low-rank pass of projection(s) over every slot, from the
  // independent per-expert factors (no sharing across grid rows or columns):
  //   zpe = Sigma * (V_pe[e]^T B[slot])   then   out[slot] += U_pe[e] zpe
  // Both products are grouped over all experts' tiles in one launch each, with
  // the fused path's tuning: split-K warp-level MMA below 256 tokens (the z
  // splits reduced by the last CTA of a tile), the dense tcgen05 kernel above.
  auto per_expert_lr = [&](int np, const int *projs, const __half *bsrc, int ldb, const int *b_row,
                           float *const *outs, int ldo, const GemmPlan &zp) -> tileq_status {
    const GemmPlan &up = plan.pe_u;
    bool tc = zp.tc;  // the dense tcgen05 kernel takes K in multiples of 64 (the U side: K = rank)
    for (int i = 0; i < np; ++i) tc = tc && li.p[projs[i]].rank % 64 == 0;
    if (tc) {
      for (int i = 0; i < np; ++i) {
        const ProjInfo &q = li.p[projs[i]];
        int8_t ident[kMaxExperts];
        for (int e = 0; e < kMaxExperts; ++e) ident[e] = (int8_t)e;
        TcF16 z;
        z.arow[0] = at<__half>(packed_pe, ppl.vr[projs[i]]);
        z.lda = q.d_in;
        z.arows = K * pad128(q.rank);
        z.d_out = q.rank;
        z.d_in = q.d_in;
        z.tiles = at<int4>(ws, w.tiles_main);
        z.tile_count = at<int>(ws, w.tile_counts);
        z.a_blk = ident;
        z.b = bsrc;
        z.brows = plan.P;
        z.ldb = ldb;
        z.epi = EPI_STORE_F16;
        z.out[0] = at<__half>(ws, w.zpe[i]);
        z.ldo = q.rank;
        z.col_scale[0] = layer->proj[projs[i]].Sigma;
        if ((st = tc_f16(z, zp, ws, w, stream)) != TILEQ_OK) return st;
        TcF16 u;
        u.arow[0] = at<__half>(packed_pe, ppl.ur[projs[i]]);
        u.lda = q.rank;
        u.arows = K * pad128(q.d_out);
        u.d_out = q.d_out;
        u.d_in = q.rank;
        u.tiles = z.tiles;
        u.tile_count = z.tile_count;
        u.a_blk = ident;
        u.b = at<__half>(ws, w.zpe[i]);
        u.brows = plan.P;
        u.ldb = q.rank;
        u.epi = EPI_ACCUM_F32;
        u.out[0] = outs[i];
        u.ldo = ldo;
        if ((st = tc_f16(u, up, ws, w, stream)) != TILEQ_OK) return st;
      }
      return TILEQ_OK;
    }
    GemmBatch zb, ub;
    const int ncnt = zp.slots * zp.m_tiles;  // split-K arrival counters of one problem
    for (int i = 0; i < np; ++i) {
      const ProjInfo &q = li.p[projs[i]];
      zb.p[i] = problem(zp, ws, w);
      GemmProblem &z = zb.p[i];
      z.tiles = at<int4>(ws, w.tiles_main);
      z.tile_count = at<int>(ws, w.tile_counts);
      z.d_out = q.rank;
      z.d_in = q.d_in;
      z.a[0] = at<uint4>(packed_pe, ppl.vf[projs[i]]);
      z.b = bsrc;
      z.ldb = ldb;
      z.b_row = b_row;
      z.epi = EPI_STORE_F16;
      z.col_scale = layer->proj[projs[i]].Sigma;
      z.out[0] = at<__half>(ws, w.zpe[i]);
      z.ldo = q.rank;
      z.counters = at<int>(ws, w.counters) + i * ncnt;
      z.part = at<float>(ws, w.part) + (size_t)i * (zp.part_floats() / std::max(1, zp.np));
      if (!b_row) tma_b(z, plan.P, zp.bn);
      ub.p[i] = problem(up, ws, w);
      GemmProblem &u = ub.p[i];
      u.m_tiles = cdiv(q.d_out, 128);
      u.tiles = z.tiles;
      u.tile_count = z.tile_count;
      u.d_out = q.d_out;
      u.d_in = q.rank;
      u.a[0] = at<uint4>(packed_pe, ppl.uf[projs[i]]);
      u.b = at<__half>(ws, w.zpe[i]);
      u.ldb = q.rank;
      u.epi = EPI_ACCUM_F32;
      u.out[0] = outs[i];
      u.ldo = ldo;
      tma_b(u, plan.P, up.bn);
    }
    if ((st = gemm(zb, np, 1, zp, stream)) != TILEQ_OK) return st;
    return gemm(ub, np, 1, up, stream);
  };

  if (layer->kind == TILEQ_LINEAR) {
    const ProjInfo &q = li.p[0];
    ScaleGatherArgs sg{plan.P, q.d_in, w.ld_x, at<int>(ws, w.slot_tok), at<float>(ws, w.slot_w),
                       at<__half>(ws, w.x16), xext};
    TQ_CUDA(launch_pdl(scale_gather_kernel, dim3(nblocks((long long)plan.P * (q.d_in / 2), 256)), dim3(256), 0, stream, sg));
    TQ_LAUNCHED();
    Residual r;
    r.b = xext;
    r.ldb = w.ld_x;
    r.out[0] = at<float>(ws, w.ybuf);
    r.ldo = q.d_out;
    if ((st = run_residual(r, plan.linear, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    if (q.rank > 0) {
      const int projs[1] = {0};
      float *outs[1] = {at<float>(ws, w.ybuf)};
      st = per_expert_lr(1, projs, xext, w.ld_x, nullptr, outs, q.d_out, plan.pe_zx);
      if (st != TILEQ_OK) return st;
    }
    for (int sidx = ST_ZPROJ; sidx <= ST_ZDOWN; ++sidx) mark(sidx, stream);
  } else {
    const ProjInfo &qg = li.p[0], &qd = li.p[2];
    const int D = layer->d_model, F = layer->d_ff;
    __half *hext = at<__half>(ws, w.hext);
    GatherExtArgs ga;
    std::memset(&ga, 0, sizeof(ga));
    ga.P = plan.P;
    ga.d = D;
    ga.r = qg.rank;
    ga.ld = w.ld_x;
    ga.slot_tok = at<int>(ws, w.slot_tok);
    ga.x16 = at<__half>(ws, w.x16);
    ga.out = xext;
    ga.T = T;
    ga.k = top_k;
    ga.slot_of_pair = at<int>(ws, w.slot_of_pair);
    ga.status = at<int>(ws, w.status);
    TQ_CUDA(launch_pdl(gather_ext_kernel, dim3(gather_blocks((long long)T * (D / 8))), dim3(256), 0, stream, ga));
    TQ_LAUNCHED();
    Residual r;
    r.np = 2;
    r.proj[1] = 1;
    r.b = xext;
    r.ldb = w.ld_x;
    r.epi = EPI_STORE2_F32;
    r.out[0] = at<float>(ws, w.g32);
    r.out[1] = at<float>(ws, w.u32);
    r.ldo = F;
    if ((st = run_residual(r, plan.gateup, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    if (qg.rank > 0) {
      const int projs[2] = {0, 1};
      float *outs[2] = {at<float>(ws, w.g32), at<float>(ws, w.u32)};
      st = per_expert_lr(2, projs, xext, w.ld_x, nullptr, outs, F, plan.pe_zx);
      if (st != TILEQ_OK) return st;
    }
    mark(ST_ZPROJ, stream);
    SwigluArgs sa{(long long)plan.P * F, F, w.ld_h, at<float>(ws, w.g32), at<float>(ws, w.u32),
                  at<float>(ws, w.slot_w), hext, at<int>(ws, w.status)};
    TQ_CUDA(launch_pdl(swiglu_kernel, dim3(nblocks(sa.n, 256)), dim3(256), 0, stream, sa));
    TQ_LAUNCHED();
    mark(ST_GATEUP, stream);
    Residual rd;
    rd.proj[0] = 2;
    rd.b = hext;
    rd.ldb = w.ld_h;
    rd.out[0] = at<float>(ws, w.ybuf);
    rd.ldo = D;
    if ((st = run_residual(rd, plan.down, li, pl, packed, ws, w, stream)) != TILEQ_OK) return st;
    if (qd.rank > 0) {
      const int projs[1] = {2};
      float *outs[1] = {at<float>(ws, w.ybuf)};
      st = per_expert_lr(1, projs, hext, w.ld_h, nullptr, outs, D, plan.pe_zd);
      if (st != TILEQ_OK) return st;
    }
    mark(ST_ZDOWN, stream);
  }
  const float *yshared = nullptr;
  if ((st = run_shared(layer, pl, w, packed, ws, T, &yshared, stream)) != TILEQ_OK) return st;
  mark(ST_SHARED, stream);
  mark(ST_RESIDUAL, stream);
  if ((st = run_combine(li, w, ws, T, top_k, yshared, out, stream)) != TILEQ_OK) return st;
  mark(ST_COMBINE, stream);
  return copy_route_out(layer, w, ws, T, top_k, route, stream);
}

tileq_status tileq_route(const float *router_logits, int T, int K, int top_k, tileq_route_out *route,
                         void *ws, size_t ws_bytes, tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (T < 0 || K < 1 || K > kMaxExperts || top_k < 1 || top_k > K || top_k > kMaxTopK)
    return TILEQ_ERR_INVALID_ARG;
  if (!route || !route->topk_idx || !route->topk_w || !route->expert_offsets || !route->sorted_pairs)
    return TILEQ_ERR_INVALID_ARG;
  if (T == 0) return TILEQ_OK;
  if (!router_logits || !ws) return TILEQ_ERR_INVALID_ARG;
  // routing-only layout: a minimal linear layer of K experts on a K x 1 grid
  tileq_layer L;
  std::memset(&L, 0, sizeof(L));
  L.kind = TILEQ_LINEAR;
  L.K = K;
  L.M = K;
  L.N = 1;
  int32_t grid[kMaxExperts];
  for (int e = 0; e < K; ++e) grid[e] = e;
  L.proj[0].d_in = 128;
  L.proj[0].d_out = 16;
  L.proj[0].group = 128;
  L.proj[0].grid_assign = grid;
  LayerInfo li;
  tileq_status st = validate_layer(&L, &li, false);
  if (st != TILEQ_OK) return st;
  const WsLayout w = ws_layout(&L, li, T, top_k, true);
  if (ws_bytes < w.total) return TILEQ_ERR_WORKSPACE;
  const int zids[2] = {0, 0};
  st = run_route_permute(&L, li, w, nullptr, T, router_logits, top_k, ws, 0, zids, -1, stream);
  if (st != TILEQ_OK) return st;
  return copy_route_out(&L, w, ws, T, top_k, route, stream);
}

tileq_status tileq_device_status(void *ws, int *status, tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!ws || !status) return TILEQ_ERR_INVALID_ARG;
  int h = 0;
  TQ_CUDA(cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, stream));
  TQ_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), stream));
  TQ_CUDA(cudaStreamSynchronize(stream));
  *status = h;
  return TILEQ_OK;
}

tileq_status tileq_set_stage_events(void **events, int n_events) {
  if (events == nullptr || n_events <= 0) {
    g_n_stage_events = 0;
    return TILEQ_OK;
  }
  if (n_events > 16) return TILEQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i) {
    if (!events[i]) return TILEQ_ERR_INVALID_ARG;
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_n_stage_events = n_events;
  return TILEQ_OK;
}

tileq_status tileq_launch_count(unsigned long long *count) {
  if (!count) return TILEQ_ERR_INVALID_ARG;
  *count = g_launches.load();
  return TILEQ_OK;
}

tileq_status tileq_selftest_bounded_wait(void *ws, size_t ws_bytes, int max_polls,
                                         tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!ws || ws_bytes < 256 || max_polls < 0 || max_polls > (1 << 24)) return TILEQ_ERR_INVALID_ARG;
  bounded_wait_kernel<<<1, 32, 0, stream>>>(static_cast<int *>(ws), max_polls);
  TQ_LAUNCHED();
  return TILEQ_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free routing
// tileq_route_static runs the same route and permute kernels as tileq_route,
// but its scratch is this file's static device array instead of a
// caller-supplied workspace, so a caller needs no device allocation at all.
namespace {

constexpr size_t kRouteStaticBytes = (size_t)6 << 20;  // 6 MiB per device
constexpr int kRouteStaticDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kRouteStaticBytes];

std::mutex g_route_static_mu;
void *g_route_static_ptr[kRouteStaticDevices] = {};

// Set-up, once per device with that device current: look up the address of
// the static scratch and zero it (the status word and the split-K counters of
// the workspace layout must start at zero).  Runs synchronously, so the first
// call on a device must not be made while a stream is being captured.
tileq_status route_static_scratch(void **ptr) {
  int dev = -1;
  TQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kRouteStaticDevices) return TILEQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_route_static_mu);
  if (g_route_static_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return TILEQ_ERR_CUDA;
    TQ_CUDA(cudaMemset(p, 0, kRouteStaticBytes));
    TQ_CUDA(cudaDeviceSynchronize());
    g_route_static_ptr[dev] = p;
  }
  *ptr = g_route_static_ptr[dev];
  return TILEQ_OK;
}

}  // namespace

extern "C" tileq_status tileq_route_static(const float *router_logits, int T, int K, int top_k,
                                           tileq_route_out *route, tileq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (T < 0 || K < 1 || K > kMaxExperts || top_k < 1 || top_k > K || top_k > kMaxTopK)
    return TILEQ_ERR_INVALID_ARG;
  if (!route || !route->topk_idx || !route->topk_w || !route->expert_offsets || !route->sorted_pairs)
    return TILEQ_ERR_INVALID_ARG;
  if ((long long)T * top_k > TILEQ_ROUTE_STATIC_MAX_PAIRS) return TILEQ_ERR_UNSUPPORTED;
  if (T == 0) return TILEQ_OK;
  if (!router_logits) return TILEQ_ERR_INVALID_ARG;
  // the same routing-only layout as tileq_route: K experts on a K x 1 grid
  tileq_layer L;
  std::memset(&L, 0, sizeof(L));
  L.kind = TILEQ_LINEAR;
  L.K = K;
  L.M = K;
  L.N = 1;
  int32_t grid[kMaxExperts];
  for (int e = 0; e < K; ++e) grid[e] = e;
  L.proj[0].d_in = 128;
  L.proj[0].d_out = 16;
  L.proj[0].group = 128;
  L.proj[0].grid_assign = grid;
  LayerInfo li;
  tileq_status st = validate_layer(&L, &li, false);
  if (st != TILEQ_OK) return st;
  const WsLayout w = ws_layout(&L, li, T, top_k, true);
  if (w.total > kRouteStaticBytes) return TILEQ_ERR_UNSUPPORTED;
  void *ws = nullptr;
  if ((st = route_static_scratch(&ws)) != TILEQ_OK) return st;
  const int zids[2] = {0, 0};
  st = run_route_permute(&L, li, w, nullptr, T, router_logits, top_k, ws, 0, zids, -1, stream);
  if (st != TILEQ_OK) return st;
  return copy_route_out(&L, w, ws, T, top_k, route, stream);
}

namespace tileq {
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n); }
void mark_stage(int stage, cudaStream_t stream) { mark(stage, stream); }
bool tensor_map_2b(CUtensorMap *m, const void *base, int rows, int cols, int ld, int box_rows) {
  return make_map(m, base, rows, cols, ld, box_rows);
}
int dense_tile_items(int items, int m_units) { return dense_bn(items, m_units); }
}  // namespace tileq
