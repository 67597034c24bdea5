// C ABI of the TileQ MoE forward (include/tileq.h): host-side validation,
// packed-weight and workspace layouts, and the launch sequence.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <vector>

#include "kernels.cuh"

using namespace tileq;

namespace tileq {
void count_launches(int n);
}

namespace {

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }
int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

struct ProjInfo {
  int d_in, d_out, rank, group, G;
  int8_t m_of[kMaxExperts], n_of[kMaxExperts];
};

struct LayerInfo {
  int nproj;
  ProjInfo p[3];
  int d_x, d_y;
};

tileq_status validate_layer(const tileq_layer *L, LayerInfo *li, bool need_device_ptrs = true) {
  if (!L) return TILEQ_ERR_INVALID_ARG;
  if (L->kind != TILEQ_LINEAR && L->kind != TILEQ_SWIGLU) return TILEQ_ERR_INVALID_ARG;
  if (L->K < 1 || L->M < 1 || L->N < 1 || (long long)L->M * L->N < L->K) return TILEQ_ERR_INVALID_ARG;
  if (L->K > kMaxExperts || L->M > kMaxExperts || L->N > kMaxExperts) return TILEQ_ERR_UNSUPPORTED;
  li->nproj = L->kind == TILEQ_LINEAR ? 1 : 3;
  for (int pi = 0; pi < li->nproj; ++pi) {
    const tileq_proj &p = L->proj[pi];
    ProjInfo &q = li->p[pi];
    if (p.d_in <= 0 || p.d_out <= 0 || p.rank < 0 || p.group <= 0) return TILEQ_ERR_INVALID_ARG;
    if (p.d_out % 16 || p.d_in % 128 || p.group % 32 || p.d_in % p.group || p.rank % 16 ||
        p.rank > 256)
      return TILEQ_ERR_UNSUPPORTED;
    if (!p.grid_assign) return TILEQ_ERR_INVALID_ARG;
    if (need_device_ptrs) {
      if (!p.codes || !p.scales || !p.zeros) return TILEQ_ERR_INVALID_ARG;
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
  }
  if (L->kind == TILEQ_SWIGLU) {
    const ProjInfo &g = li->p[0], &u = li->p[1], &d = li->p[2];
    if (g.d_in != L->d_model || g.d_out != L->d_ff || u.d_in != L->d_model || u.d_out != L->d_ff ||
        d.d_in != L->d_ff || d.d_out != L->d_model)
      return TILEQ_ERR_INVALID_ARG;
    if (g.rank != u.rank) return TILEQ_ERR_UNSUPPORTED;
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

// ------------------------------------------------------------------ packed layout
struct PackedLayout {
  size_t qw[3], sz[3], uf[3], vf[3], sh[3], total;
};

PackedLayout packed_layout(const tileq_layer *L, const LayerInfo &li) {
  PackedLayout pl{};
  size_t off = 0;
  for (int p = 0; p < li.nproj; ++p) {
    const ProjInfo &q = li.p[p];
    pl.qw[p] = off;
    off += align_up((size_t)L->K * q.d_out * q.d_in / 4);
    pl.sz[p] = off;
    off += align_up((size_t)L->K * q.d_out * q.G * 4);
    pl.uf[p] = off;
    off += align_up((size_t)L->M * q.d_out * q.rank * 2);
    pl.vf[p] = off;
    off += align_up((size_t)L->N * q.d_in * q.rank * 2);
  }
  for (int i = 0; i < 3; ++i) {
    pl.sh[i] = off;
    off += align_up((size_t)L->shared_d_ff * L->d_model * 2);
  }
  pl.total = off;
  return pl;
}

struct PePackedLayout {
  size_t uf[3], vf[3], total;
};

PePackedLayout pe_layout(const tileq_layer *L, const LayerInfo &li) {
  PePackedLayout pl{};
  size_t off = 0;
  for (int p = 0; p < li.nproj; ++p) {
    const ProjInfo &q = li.p[p];
    pl.uf[p] = off;
    off += align_up((size_t)L->K * q.d_out * q.rank * 2);
    pl.vf[p] = off;
    off += align_up((size_t)L->K * q.d_in * q.rank * 2);
  }
  pl.total = off;
  return pl;
}

// ------------------------------------------------------------------ workspace layout
struct WsLayout {
  int P, bn, ksplit, slots_main, slots_z;
  size_t status, topk_idx, topk_w, expert_offsets, sorted_pairs, slot_of_pair, slot_tok, slot_w,
      dest, tiles_main, tile_first, tile_counts;
  size_t col_offsets[2], colpair_tok[2], zidx[2], tiles_z[2];
  size_t row_offsets, rowpair_tok, rowpair_row, aidx;
  size_t x16, xs, zc[2], zs, abuf, h, ybuf, hs, ys, g32, u32, zpe[2];
  size_t total;
};

int choose_bn(int P, int K) {
  const int avg = P / std::max(1, K);
  if (avg <= 8) return 8;
  if (avg <= 16) return 16;
  if (avg <= 32) return 32;
  return 64;
}

WsLayout ws_layout(const tileq_layer *L, const LayerInfo &li, int T, int k) {
  WsLayout w{};
  const int P = T * k;
  w.P = P;
  w.bn = choose_bn(P, L->K);
  w.slots_main = cdiv(P, w.bn) + L->K;
  w.slots_z = cdiv(P, w.bn) + L->N;
  {
    // split K of the last (combined) GEMM until the grid covers ~2 waves of 148 SMs
    const ProjInfo &q = li.p[li.nproj - 1];
    const long long ctas = (long long)(std::min(L->K, P) + P / w.bn) * cdiv(q.d_out, 64);
    const int nkb = q.d_in / 128;
    int ks = (int)std::max(1LL, (2LL * 148 + ctas - 1) / std::max(1LL, ctas));
    ks = std::min(ks, std::max(1, nkb / 4));
    w.ksplit = std::max(1, std::min(ks, 8));
  }
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
  w.tiles_main = take((size_t)w.slots_main * 16);
  w.tile_first = take((L->K + 1) * 4);
  w.tile_counts = take(16);
  for (int z = 0; z < 2; ++z) {
    w.col_offsets[z] = take((L->N + 1) * 4);
    w.colpair_tok[z] = take(Pz * 4);
    w.zidx[z] = take(Pz * 4);
    w.tiles_z[z] = take((size_t)w.slots_z * 16);
  }
  w.row_offsets = take((L->M + 1) * 4);
  w.rowpair_tok = take(Pz * 4);
  w.rowpair_row = take(Pz * 4);
  w.aidx = take(Pz * 4);
  w.x16 = take((size_t)std::max(T, 1) * li.d_x * 2);
  const int rmax = std::max(std::max(li.p[0].rank, li.nproj > 1 ? li.p[1].rank : 0),
                            li.p[li.nproj - 1].rank);
  if (L->kind == TILEQ_LINEAR) {
    w.xs = take(Pz * li.d_x * 2);
    w.zc[0] = take(Pz * li.p[0].rank * 2);
    w.abuf = take(Pz * li.p[0].rank * 2);
  } else {
    w.zc[0] = take(Pz * li.p[0].rank * 2);
    w.zc[1] = take(Pz * li.p[1].rank * 2);
    w.zs = take(Pz * li.p[2].rank * 4);
    w.abuf = take(Pz * li.p[2].rank * 2);
    w.h = take(Pz * L->d_ff * 2);
    w.g32 = take(Pz * L->d_ff * 4);
    w.u32 = take(Pz * L->d_ff * 4);
  }
  w.zpe[0] = take(Pz * rmax * 2);
  w.zpe[1] = take(Pz * rmax * 2);
  w.ybuf = take((size_t)w.ksplit * Pz * li.d_y * 4);
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

GemmProblem problem() {
  GemmProblem g;
  std::memset(&g, 0, sizeof(g));
  g.only_group = -1;
  g.ksplit = 1;
  return g;
}

#define TQ_CUDA(call)                                       \
  do {                                                      \
    if ((call) != cudaSuccess) return TILEQ_ERR_CUDA;       \
  } while (0)

#define TQ_LAUNCHED()                                       \
  do {                                                      \
    count_launches();                                       \
    if (cudaGetLastError() != cudaSuccess) return TILEQ_ERR_CUDA; \
  } while (0)

std::atomic<unsigned long long> g_launches{0};
cudaEvent_t g_stage_events[16];
int g_n_stage_events = 0;

// Stage boundaries of one forward (see tileq_set_stage_events).
enum Stage { ST_BEGIN = 0, ST_ROUTE, ST_PERMUTE, ST_ZPROJ, ST_GATEUP, ST_ZDOWN, ST_ROWACC,
             ST_RESIDUAL, ST_SHARED, ST_COMBINE };

void mark(int stage, cudaStream_t stream) {
  if (stage < g_n_stage_events) cudaEventRecord(g_stage_events[stage], stream);
}

unsigned nblocks(long long n, int per) { return (unsigned)((n + per - 1) / per); }

// Residual projection problem for the Q2 GEMM: A = packed codes of projection p.
GemmProblem residual_problem(const tileq_layer *L, const LayerInfo &li, const PackedLayout &pl,
                             const void *packed, int p) {
  const ProjInfo &q = li.p[p];
  GemmProblem g = problem();
  g.d_out = q.d_out;
  g.d_in = q.d_in;
  g.group_size = q.group;
  g.a[0] = at<uint4>(packed, pl.qw[p]);
  g.sz[0] = at<uint32_t>(packed, pl.sz[p]);
  g.a_stride = (long long)(q.d_out / 16) * (q.d_in / 128) * 32;
  g.sz_stride = (long long)(q.d_out / 16) * q.G * 16;
  g.m_tiles = cdiv(q.d_out, 64);
  (void)L;
  return g;
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
  ra.topk_idx = at<int32_t>(ws, w.topk_idx);
  ra.topk_w = at<float>(ws, w.topk_w);
  mark(ST_BEGIN, stream);
  route_kernel<<<nblocks(T, 8), 256, 0, stream>>>(ra);
  TQ_LAUNCHED();
  mark(ST_ROUTE, stream);

  PermuteArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  pa.T = T;
  pa.k = top_k;
  pa.K = L->K;
  pa.M = L->M;
  pa.N = L->N;
  pa.bn = w.bn;
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
  pa.n_zproj = n_zproj;
  for (int z = 0; z < 2; ++z) {
    if (z < n_zproj) std::memcpy(pa.n_of[z], li.p[zproj_ids[z]].n_of, kMaxExperts);
    pa.col_offsets[z] = at<int>(ws, w.col_offsets[z]);
    pa.colpair_tok[z] = at<int>(ws, w.colpair_tok[z]);
    pa.zidx[z] = at<int>(ws, w.zidx[z]);
    pa.tiles_z[z] = at<int4>(ws, w.tiles_z[z]);
  }
  pa.row_proj = row_proj;
  if (row_proj >= 0) std::memcpy(pa.m_of_row, li.p[row_proj].m_of, kMaxExperts);
  pa.row_offsets = at<int>(ws, w.row_offsets);
  pa.rowpair_tok = at<int>(ws, w.rowpair_tok);
  pa.rowpair_row = at<int>(ws, w.rowpair_row);
  pa.aidx = at<int>(ws, w.aidx);
  permute_kernel<<<1, 1024, 0, stream>>>(pa);
  TQ_LAUNCHED();
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

tileq_status run_shared_and_combine(const tileq_layer *L, const LayerInfo &li,
                                    const PackedLayout &pl, const WsLayout &w, const void *packed,
                                    void *ws, int T, int top_k, void *out, cudaStream_t stream) {
  const float *yshared = nullptr;
  if (L->shared_d_ff > 0) {
    const int Fs = L->shared_d_ff, D = L->d_model;
    const int bn = T <= 8 ? 8 : T <= 16 ? 16 : T <= 32 ? 32 : 64;
    GemmBatch b;
    b.p[0] = problem();
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
    g.m_tiles = cdiv(Fs, 64);
    if (launch_gemm(b, 1, GemmShape{AM_F16, 2, bn, 4}, cdiv(T, bn), stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    GemmProblem &d = b.p[0];
    d = problem();
    d.static_items = T;
    d.d_out = D;
    d.d_in = Fs;
    d.a[0] = at<uint4>(packed, pl.sh[2]);
    d.b = at<__half>(ws, w.hs);
    d.ldb = Fs;
    d.epi = EPI_STORE_F32;
    d.out[0] = at<float>(ws, w.ys);
    d.ldo = D;
    d.m_tiles = cdiv(D, 64);
    if (launch_gemm(b, 1, GemmShape{AM_F16, 1, bn, 4}, cdiv(T, bn), stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    yshared = at<float>(ws, w.ys);
  }
  mark(ST_SHARED, stream);
  CombineArgs ca;
  ca.T = T;
  ca.k = top_k;
  ca.d = li.d_y;
  ca.ksplit = w.ksplit;
  ca.split_stride = (long long)w.P * li.d_y;
  ca.slot_of_pair = at<int>(ws, w.slot_of_pair);
  ca.ybuf = at<float>(ws, w.ybuf);
  ca.yshared = yshared;
  ca.out = static_cast<__nv_bfloat16 *>(out);
  combine_kernel<<<nblocks((long long)T * (li.d_y / 4), 256), 256, 0, stream>>>(ca);
  TQ_LAUNCHED();
  mark(ST_COMBINE, stream);
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
  if ((long long)T * top_k > (1LL << 28)) return TILEQ_ERR_UNSUPPORTED;
  const WsLayout w = ws_layout(layer, *li, T, top_k);
  if (ws_bytes < w.total) return TILEQ_ERR_WORKSPACE;
  return TILEQ_OK;
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
      const long long n = (long long)K * (q.d_out / 16) * (q.d_in / 128) * 32;
      pack_codes_kernel<<<nblocks(n, 256), 256, 0, stream>>>(src.codes, at<uint4>(packed, pl.qw[p]),
                                                              K, q.d_out, q.d_in);
      TQ_LAUNCHED();
    }
    {
      const long long n = (long long)K * q.d_out * q.G;
      pack_sz_kernel<<<nblocks(n, 256), 256, 0, stream>>>(static_cast<const __half *>(src.scales),
                                                           src.zeros, at<uint32_t>(packed, pl.sz[p]),
                                                           K, q.d_out, q.G);
      TQ_LAUNCHED();
    }
    if (q.rank > 0) {
      const __nv_bfloat16 *U = static_cast<const __nv_bfloat16 *>(src.U);
      const __nv_bfloat16 *V = static_cast<const __nv_bfloat16 *>(src.V);
      // U block m: rows o (d_out), cols i (rank): element at U[(m*d_out + o)*rank + i]
      long long n = (long long)layer->M * (q.d_out / 16) * (q.rank / 16) * 32;
      pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(U, (long long)q.d_out * q.rank, q.rank, 1,
                                                             layer->M, q.d_out, q.rank,
                                                             at<uint4>(packed, pl.uf[p]));
      TQ_LAUNCHED();
      // V_n^T: rows i (rank), cols k (d_in): element at V[(n*d_in + k)*rank + i]
      n = (long long)layer->N * (q.rank / 16) * (q.d_in / 16) * 32;
      pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(V, (long long)q.d_in * q.rank, 1, q.rank,
                                                             layer->N, q.rank, q.d_in,
                                                             at<uint4>(packed, pl.vf[p]));
      TQ_LAUNCHED();
    }
  }
  if (layer->shared_d_ff > 0) {
    const int Fs = layer->shared_d_ff, D = layer->d_model;
    for (int i = 0; i < 3; ++i) {
      const int R = i < 2 ? Fs : D, Cc = i < 2 ? D : Fs;
      const long long n = (long long)(R / 16) * (Cc / 16) * 32;
      pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16 *>(layer->shared_w[i]), 0, Cc, 1, 1, R, Cc,
          at<uint4>(packed, pl.sh[i]));
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
  const int K = layer->K;

  if (layer->kind == TILEQ_LINEAR) {
    const ProjInfo &q = li.p[0];
    const int zids[2] = {0, 0};
    st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, q.rank > 0 ? 1 : 0, zids,
                           q.rank > 0 ? 0 : -1, stream);
    if (st != TILEQ_OK) return st;
    ScaleGatherArgs sg{w.P, q.d_in, at<int>(ws, w.slot_tok), at<float>(ws, w.slot_w),
                       at<__half>(ws, w.x16), at<__half>(ws, w.xs)};
    scale_gather_kernel<<<nblocks((long long)w.P * (q.d_in / 2), 256), 256, 0, stream>>>(sg);
    TQ_LAUNCHED();
    if (q.rank > 0) {
      GemmBatch b;
      b.p[0] = problem();
      GemmProblem &z = b.p[0];
      z.tiles = at<int4>(ws, w.tiles_z[0]);
      z.tile_count = at<int>(ws, w.tile_counts) + 1;
      z.d_out = q.rank;
      z.d_in = q.d_in;
      z.a[0] = at<uint4>(packed, pl.vf[0]);
      z.a_stride = (long long)(q.rank / 16) * (q.d_in / 16) * 32;
      z.b = at<__half>(ws, w.x16);
      z.ldb = q.d_in;
      z.b_row = at<int>(ws, w.colpair_tok[0]);
      z.epi = EPI_STORE_F16;
      z.col_scale = layer->proj[0].Sigma;
      z.out[0] = at<__half>(ws, w.zc[0]);
      z.ldo = q.rank;
      z.m_tiles = cdiv(q.rank, 64);
      if (launch_gemm(b, 1, GemmShape{AM_F16, 1, w.bn, 4}, w.slots_z, stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
      mark(ST_ZPROJ, stream);
      mark(ST_GATEUP, stream);
      mark(ST_ZDOWN, stream);
      LrAccArgs la;
      std::memset(&la, 0, sizeof(la));
      la.k = top_k;
      la.r = q.rank;
      la.row_offsets = at<int>(ws, w.row_offsets);
      la.M = layer->M;
      la.rowpair_tok = at<int>(ws, w.rowpair_tok);
      la.rowpair_row = at<int>(ws, w.rowpair_row);
      la.topk_idx = at<int32_t>(ws, w.topk_idx);
      la.topk_w = at<float>(ws, w.topk_w);
      std::memcpy(la.m_of, q.m_of, kMaxExperts);
      la.slot_of_pair = at<int>(ws, w.slot_of_pair);
      la.zcol = at<__half>(ws, w.zc[0]);
      la.zidx = at<int>(ws, w.zidx[0]);
      la.a = at<__half>(ws, w.abuf);
      lr_accumulate_kernel<<<nblocks((long long)w.P * q.rank, 256), 256, 0, stream>>>(la);
      TQ_LAUNCHED();
    } else {
      mark(ST_ZPROJ, stream);
      mark(ST_GATEUP, stream);
      mark(ST_ZDOWN, stream);
    }
    mark(ST_ROWACC, stream);
    GemmBatch b;
    b.p[0] = residual_problem(layer, li, pl, packed, 0);
    GemmProblem &g = b.p[0];
    g.tiles = at<int4>(ws, w.tiles_main);
    g.tile_count = at<int>(ws, w.tile_counts);
    g.b = at<__half>(ws, w.xs);
    g.ldb = q.d_in;
    g.rank = q.rank;
    if (q.rank > 0) {
      g.u[0] = at<uint4>(packed, pl.uf[0]);
      g.u_stride = (long long)(q.d_out / 16) * (q.rank / 16) * 32;
      std::memcpy(g.u_blk[0], q.m_of, kMaxExperts);
      g.zb[0] = at<__half>(ws, w.abuf);
      g.ldz = q.rank;
      g.z_row[0] = at<int>(ws, w.aidx);
    }
    g.epi = EPI_STORE_F32;
    g.out[0] = at<float>(ws, w.ybuf);
    g.ldo = q.d_out;
    g.out_split_stride = (long long)w.P * q.d_out;
    g.ksplit = w.ksplit;
    if (launch_gemm(b, 1, GemmShape{AM_Q2, 1, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    mark(ST_RESIDUAL, stream);
  } else {
    const ProjInfo &qg = li.p[0], &qd = li.p[2];
    const int zids[2] = {0, 1};
    const bool lr_gu = qg.rank > 0, lr_d = qd.rank > 0;
    st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, lr_gu ? 2 : 0, zids,
                           lr_d ? 2 : -1, stream);
    if (st != TILEQ_OK) return st;
    const int D = layer->d_model, F = layer->d_ff;
    if (lr_gu) {
      // z_{t,n} = Sigma * (V_n^T x_t) once per distinct (token, grid column), gate and up
      GemmBatch b;
      for (int p = 0; p < 2; ++p) {
        const ProjInfo &q = li.p[p];
        b.p[p] = problem();
        GemmProblem &z = b.p[p];
        z.tiles = at<int4>(ws, w.tiles_z[p]);
        z.tile_count = at<int>(ws, w.tile_counts) + 1 + p;
        z.d_out = q.rank;
        z.d_in = D;
        z.a[0] = at<uint4>(packed, pl.vf[p]);
        z.a_stride = (long long)(q.rank / 16) * (D / 16) * 32;
        z.b = at<__half>(ws, w.x16);
        z.ldb = D;
        z.b_row = at<int>(ws, w.colpair_tok[p]);
        z.epi = EPI_STORE_F16;
        z.col_scale = layer->proj[p].Sigma;
        z.out[0] = at<__half>(ws, w.zc[p]);
        z.ldo = q.rank;
        z.m_tiles = cdiv(q.rank, 64);
      }
      if (launch_gemm(b, 2, GemmShape{AM_F16, 1, w.bn, 4}, w.slots_z, stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
    }
    mark(ST_ZPROJ, stream);
    {
      // gate/up residual + U_m z (K extension) + SwiGLU, h = w * silu(g) * u per slot
      GemmBatch b;
      b.p[0] = residual_problem(layer, li, pl, packed, 0);
      GemmProblem &g = b.p[0];
      g.a[1] = at<uint4>(packed, pl.qw[1]);
      g.sz[1] = at<uint32_t>(packed, pl.sz[1]);
      g.tiles = at<int4>(ws, w.tiles_main);
      g.tile_count = at<int>(ws, w.tile_counts);
      g.b = at<__half>(ws, w.x16);
      g.ldb = D;
      g.b_row = at<int>(ws, w.slot_tok);
      g.rank = qg.rank;
      if (lr_gu) {
        for (int p = 0; p < 2; ++p) {
          g.u[p] = at<uint4>(packed, pl.uf[p]);
          std::memcpy(g.u_blk[p], li.p[p].m_of, kMaxExperts);
          g.zb[p] = at<__half>(ws, w.zc[p]);
          g.z_row[p] = at<int>(ws, w.zidx[p]);
        }
        g.u_stride = (long long)(F / 16) * (qg.rank / 16) * 32;
        g.ldz = qg.rank;
      }
      g.epi = EPI_SWIGLU_H;
      g.out[0] = at<__half>(ws, w.h);
      g.ldo = F;
      g.row_scale = at<float>(ws, w.slot_w);
      if (launch_gemm(b, 1, GemmShape{AM_Q2, 2, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
    }
    mark(ST_GATEUP, stream);
    if (lr_d) {
      // z'_slot = Sigma * (V_n^T h_slot) for the down projection, then the in-place
      // accumulation a_{t,m} = sum of the token's z' over its experts in grid row m
      GemmBatch b;
      b.p[0] = problem();
      GemmProblem &z = b.p[0];
      z.tiles = at<int4>(ws, w.tiles_main);
      z.tile_count = at<int>(ws, w.tile_counts);
      z.d_out = qd.rank;
      z.d_in = F;
      z.a[0] = at<uint4>(packed, pl.vf[2]);
      z.a_stride = (long long)(qd.rank / 16) * (F / 16) * 32;
      z.use_a_blk = 1;
      std::memcpy(z.a_blk, qd.n_of, kMaxExperts);
      z.b = at<__half>(ws, w.h);
      z.ldb = F;
      z.epi = EPI_STORE_F32;
      z.col_scale = layer->proj[2].Sigma;
      z.out[0] = at<float>(ws, w.zs);
      z.ldo = qd.rank;
      z.m_tiles = cdiv(qd.rank, 64);
      if (launch_gemm(b, 1, GemmShape{AM_F16, 1, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
      mark(ST_ZDOWN, stream);
      LrAccArgs la;
      std::memset(&la, 0, sizeof(la));
      la.k = top_k;
      la.r = qd.rank;
      la.row_offsets = at<int>(ws, w.row_offsets);
      la.M = layer->M;
      la.rowpair_tok = at<int>(ws, w.rowpair_tok);
      la.rowpair_row = at<int>(ws, w.rowpair_row);
      la.topk_idx = at<int32_t>(ws, w.topk_idx);
      la.topk_w = at<float>(ws, w.topk_w);
      std::memcpy(la.m_of, qd.m_of, kMaxExperts);
      la.slot_of_pair = at<int>(ws, w.slot_of_pair);
      la.zslot = at<float>(ws, w.zs);
      la.a = at<__half>(ws, w.abuf);
      lr_accumulate_kernel<<<nblocks((long long)w.P * qd.rank, 256), 256, 0, stream>>>(la);
      TQ_LAUNCHED();
    } else {
      mark(ST_ZDOWN, stream);
    }
    mark(ST_ROWACC, stream);
    {
      GemmBatch b;
      b.p[0] = residual_problem(layer, li, pl, packed, 2);
      GemmProblem &g = b.p[0];
      g.tiles = at<int4>(ws, w.tiles_main);
      g.tile_count = at<int>(ws, w.tile_counts);
      g.b = at<__half>(ws, w.h);
      g.ldb = F;
      g.rank = qd.rank;
      if (lr_d) {
        g.u[0] = at<uint4>(packed, pl.uf[2]);
        g.u_stride = (long long)(D / 16) * (qd.rank / 16) * 32;
        std::memcpy(g.u_blk[0], qd.m_of, kMaxExperts);
        g.zb[0] = at<__half>(ws, w.abuf);
        g.ldz = qd.rank;
        g.z_row[0] = at<int>(ws, w.aidx);
      }
      g.epi = EPI_STORE_F32;
      g.out[0] = at<float>(ws, w.ybuf);
      g.ldo = D;
      g.out_split_stride = (long long)w.P * D;
      g.ksplit = w.ksplit;
      if (launch_gemm(b, 1, GemmShape{AM_Q2, 1, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
    }
    mark(ST_RESIDUAL, stream);
  }
  (void)K;
  st = run_shared_and_combine(layer, li, pl, w, packed, ws, T, top_k, out, stream);
  if (st != TILEQ_OK) return st;
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
    long long n = (long long)K * (q.d_out / 16) * (q.rank / 16) * 32;
    pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(pe->U_pe[p]), (long long)q.d_out * q.rank, q.rank, 1, K,
        q.d_out, q.rank, at<uint4>(packed_pe, pl.uf[p]));
    TQ_LAUNCHED();
    n = (long long)K * (q.rank / 16) * (q.d_in / 16) * 32;
    pack_frag_kernel<<<nblocks(n, 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(pe->V_pe[p]), (long long)q.d_in * q.rank, 1, q.rank, K,
        q.rank, q.d_in, at<uint4>(packed_pe, pl.vf[p]));
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
  const int K = layer->K;
  const int zids[2] = {0, 0};
  st = run_route_permute(layer, li, w, x, T, router_logits, top_k, ws, 0, zids, -1, stream);
  if (st != TILEQ_OK) return st;

  // Per-expert low-rank pass of projection p over the expert's slots:
  //   zpe = Sigma * (V_pe[e]^T B[slot])  then  out[slot] += U_pe[e] zpe
  auto per_expert_lr = [&](int np, const int *projs, const __half *bsrc, int ldb, const int *b_row,
                           float *const *outs, int ldo) -> tileq_status {
    for (int e = 0; e < K; ++e) {
      GemmBatch zb, ub;
      for (int i = 0; i < np; ++i) {
        const ProjInfo &q = li.p[projs[i]];
        zb.p[i] = problem();
        GemmProblem &z = zb.p[i];
        z.tiles = at<int4>(ws, w.tiles_main);
        z.tile_count = at<int>(ws, w.tile_counts);
        z.only_group = e;
        z.group_first_tile = at<int>(ws, w.tile_first);
        z.d_out = q.rank;
        z.d_in = q.d_in;
        z.a[0] = at<uint4>(packed_pe, ppl.vf[projs[i]]);
        z.a_stride = (long long)(q.rank / 16) * (q.d_in / 16) * 32;
        z.b = bsrc;
        z.ldb = ldb;
        z.b_row = b_row;
        z.epi = EPI_STORE_F16;
        z.col_scale = layer->proj[projs[i]].Sigma;
        z.out[0] = at<__half>(ws, w.zpe[i]);
        z.ldo = q.rank;
        z.m_tiles = cdiv(q.rank, 64);
        ub.p[i] = problem();
        GemmProblem &u = ub.p[i];
        u.tiles = z.tiles;
        u.tile_count = z.tile_count;
        u.only_group = e;
        u.group_first_tile = z.group_first_tile;
        u.d_out = q.d_out;
        u.d_in = q.rank;
        u.a[0] = at<uint4>(packed_pe, ppl.uf[projs[i]]);
        u.a_stride = (long long)(q.d_out / 16) * (q.rank / 16) * 32;
        u.b = at<__half>(ws, w.zpe[i]);
        u.ldb = q.rank;
        u.epi = EPI_ACCUM_F32;
        u.out[0] = outs[i];
        u.ldo = ldo;
        u.m_tiles = cdiv(q.d_out, 64);
      }
      if (launch_gemm(zb, np, GemmShape{AM_F16, 1, w.bn, 4}, cdiv(T, w.bn), stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
      if (launch_gemm(ub, np, GemmShape{AM_F16, 1, w.bn, 4}, cdiv(T, w.bn), stream) != cudaSuccess)
        return TILEQ_ERR_CUDA;
    }
    return TILEQ_OK;
  };
  // The tiles of one expert are contiguous in the main table, from
  // tile_first[e]; the number is known only on the device, so each
  // per-expert launch covers the largest possible expert (T slots, one per
  // token) and its surplus CTAs return at once.

  if (layer->kind == TILEQ_LINEAR) {
    const ProjInfo &q = li.p[0];
    ScaleGatherArgs sg{w.P, q.d_in, at<int>(ws, w.slot_tok), at<float>(ws, w.slot_w),
                       at<__half>(ws, w.x16), at<__half>(ws, w.xs)};
    scale_gather_kernel<<<nblocks((long long)w.P * (q.d_in / 2), 256), 256, 0, stream>>>(sg);
    TQ_LAUNCHED();
    GemmBatch b;
    b.p[0] = residual_problem(layer, li, pl, packed, 0);
    GemmProblem &g = b.p[0];
    g.tiles = at<int4>(ws, w.tiles_main);
    g.tile_count = at<int>(ws, w.tile_counts);
    g.b = at<__half>(ws, w.xs);
    g.ldb = q.d_in;
    g.epi = EPI_STORE_F32;
    g.out[0] = at<float>(ws, w.ybuf);
    g.ldo = q.d_out;
    g.out_split_stride = (long long)w.P * q.d_out;
    g.ksplit = w.ksplit;
    if (launch_gemm(b, 1, GemmShape{AM_Q2, 1, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    if (q.rank > 0) {
      const int projs[1] = {0};
      float *outs[1] = {at<float>(ws, w.ybuf)};
      st = per_expert_lr(1, projs, at<__half>(ws, w.xs), q.d_in, nullptr, outs, q.d_out);
      if (st != TILEQ_OK) return st;
    }
    for (int sidx = ST_ZPROJ; sidx <= ST_RESIDUAL; ++sidx) mark(sidx, stream);
  } else {
    const ProjInfo &qg = li.p[0], &qd = li.p[2];
    const int D = layer->d_model, F = layer->d_ff;
    GemmBatch b;
    b.p[0] = residual_problem(layer, li, pl, packed, 0);
    GemmProblem &g = b.p[0];
    g.a[1] = at<uint4>(packed, pl.qw[1]);
    g.sz[1] = at<uint32_t>(packed, pl.sz[1]);
    g.tiles = at<int4>(ws, w.tiles_main);
    g.tile_count = at<int>(ws, w.tile_counts);
    g.b = at<__half>(ws, w.x16);
    g.ldb = D;
    g.b_row = at<int>(ws, w.slot_tok);
    g.epi = EPI_STORE2_F32;
    g.out[0] = at<float>(ws, w.g32);
    g.out[1] = at<float>(ws, w.u32);
    g.ldo = F;
    if (launch_gemm(b, 1, GemmShape{AM_Q2, 2, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    if (qg.rank > 0) {
      const int projs[2] = {0, 1};
      float *outs[2] = {at<float>(ws, w.g32), at<float>(ws, w.u32)};
      st = per_expert_lr(2, projs, at<__half>(ws, w.x16), D, at<int>(ws, w.slot_tok), outs, F);
      if (st != TILEQ_OK) return st;
    }
    mark(ST_ZPROJ, stream);
    SwigluArgs sa{(long long)w.P * F, F, at<float>(ws, w.g32), at<float>(ws, w.u32),
                  at<float>(ws, w.slot_w), at<__half>(ws, w.h)};
    swiglu_kernel<<<nblocks(sa.n, 256), 256, 0, stream>>>(sa);
    TQ_LAUNCHED();
    mark(ST_GATEUP, stream);
    b.p[0] = residual_problem(layer, li, pl, packed, 2);
    GemmProblem &d = b.p[0];
    d.tiles = at<int4>(ws, w.tiles_main);
    d.tile_count = at<int>(ws, w.tile_counts);
    d.b = at<__half>(ws, w.h);
    d.ldb = F;
    d.epi = EPI_STORE_F32;
    d.out[0] = at<float>(ws, w.ybuf);
    d.ldo = D;
    d.out_split_stride = (long long)w.P * D;
    d.ksplit = w.ksplit;
    if (launch_gemm(b, 1, GemmShape{AM_Q2, 1, w.bn, 4}, w.slots_main, stream) != cudaSuccess)
      return TILEQ_ERR_CUDA;
    if (qd.rank > 0) {
      const int projs[1] = {2};
      float *outs[1] = {at<float>(ws, w.ybuf)};
      st = per_expert_lr(1, projs, at<__half>(ws, w.h), F, nullptr, outs, D);
      if (st != TILEQ_OK) return st;
    }
    mark(ST_ZDOWN, stream);
    mark(ST_ROWACC, stream);
    mark(ST_RESIDUAL, stream);
  }
  st = run_shared_and_combine(layer, li, pl, w, packed, ws, T, top_k, out, stream);
  if (st != TILEQ_OK) return st;
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
  const WsLayout w = ws_layout(&L, li, T, top_k);
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

namespace tileq {
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n); }
}  // namespace tileq
