// Expert placement on the M x N tile grid: TileQ summary, section 2.1, steps
// 2-4 (feature embeddings from each expert's rank-r0 SVD factors, K-Means on
// each side that picks a preferred cell per expert, and a greedy pass that
// settles experts preferring the same cell).
//
//   pl_maxabs_kernel     per factor column, the entry of largest magnitude
//                        (64-bit atomicMax on |x| bits : ~row, so ties keep the
//                        first row); the last CTA to finish writes the
//                        columns' signs
//   pl_gram_kernel       partial fp64 Gram matrices E E^T of the sign-fixed,
//                        flattened factors, one per CTA over its slice of the
//                        flattened dimension (both sides in one launch)
//   pl_gram_sum_kernel   the partials summed in a fixed order (deterministic)
//   pl_cluster_kernel    one CTA per side: normalisation (folded into the Gram:
//                        G_ij / (|e_i| |e_j|)), farthest-first start, Lloyd
//                        iterations with every centre held as weights over the
//                        experts, so that |e_i - c_j|^2 = G_ii - 2 (G a_j)_i + a_j^T G a_j
//   pl_greedy_kernel     one CTA of two warps: the global greedy allocation,
//                        each round placing the smallest (distance, expert,
//                        cell) key over the experts' cached best free cells
//
// The factors are read twice (the sign pass and the Gram pass); everything
// after the Gram works on K x K numbers.
#include "kernels.cuh"

namespace tileq {
namespace {

constexpr int kPlMaxR0 = TILEQ_PLACE_MAX_R0;
constexpr int kPlThreads = 288;     // Gram CTA: 2 x 136 upper-triangle 4 x 4 thread tiles at K = 64
constexpr int kPlMaxCtas = 148;     // Gram CTAs per side (partials summed afterwards)
constexpr int kPlMinChunks = 4;     // at least this many tiles per Gram CTA
constexpr int kPlRowsPerCta = 1024; // factor rows per CTA of the sign pass
constexpr int kPlClusterThreads = 256;
constexpr int kPlGreedyThreads = 64;   // two warps: one lane per expert (K <= 64)

struct PlaceArgs {
  const float *f[2];          // U side, V side: [K][d][r0]
  long long d[2];             // rows of each side's factors
  int K, M, N, r0, max_iter;
  int ctas[2];                // Gram CTAs per side
  unsigned long long *keys;   // [2][K][r0]
  unsigned *ticket;           // CTAs of the sign pass that have finished
  float *sign;                // [2][K][r0]
  double *part;               // [2][kPlMaxCtas][K][K]
  double *gram;               // [2][K][K]
  int32_t *labels;            // [2][K]
  int32_t *iters;             // [2]
  int32_t *grid_assign, *ideal, *iterations;
};

// ------------------------------------------------------------ sign pass
// grid (row chunks, K, 2 sides).  A thread owns VEC consecutive columns (4 when
// r0 is a multiple of 4: 16-byte loads) and reads every step-th row of its
// chunk.  The CTA that finishes last (a ticket counter, no waiting) turns the
// keys into signs.
template <int VEC>
__device__ void maxabs_rows(const PlaceArgs &a, int s, int k, long long row0, unsigned long long *best) {
  const long long d = a.d[s];
  const int r0 = a.r0;
  const int tpr = r0 / VEC;                          // threads per row
  const int lanes = (blockDim.x / tpr) * tpr;        // threads in use: whole rows
  if ((int)threadIdx.x >= lanes) return;
  const int c0 = (threadIdx.x % tpr) * VEC;
  const int step = lanes / tpr;
  const long long row_end = row0 + kPlRowsPerCta < d ? row0 + kPlRowsPerCta : d;
  const float *f = a.f[s] + (size_t)k * d * r0 + c0;
  unsigned long long key[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) key[j] = 0ull;
#pragma unroll 8
  for (long long row = row0 + threadIdx.x / tpr; row < row_end; row += step) {
    float x[VEC];
    if constexpr (VEC == 4) {
      const float4 q = __ldg(reinterpret_cast<const float4 *>(f + row * r0));
      x[0] = q.x; x[1] = q.y; x[2] = q.z; x[3] = q.w;
    } else {
      x[0] = __ldg(f + row * r0);
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const unsigned long long kx =
          ((unsigned long long)(__float_as_uint(x[j]) & 0x7fffffffu) << 32) | (0xffffffffu - (unsigned)row);
      key[j] = kx > key[j] ? kx : key[j];
    }
  }
#pragma unroll
  for (int j = 0; j < VEC; ++j) atomicMax(&best[c0 + j], key[j]);
}

__global__ void __launch_bounds__(256) pl_maxabs_kernel(PlaceArgs a) {
  const int s = blockIdx.z, k = blockIdx.y;
  const int r0 = a.r0;
  const long long row0 = (long long)blockIdx.x * kPlRowsPerCta;
  __shared__ unsigned long long best[kPlMaxR0];
  __shared__ bool last;
  const bool work = row0 < a.d[s];
  if (work) {
    for (int c = threadIdx.x; c < r0; c += blockDim.x) best[c] = 0ull;
    __syncthreads();
    if (r0 % 4 == 0) maxabs_rows<4>(a, s, k, row0, best);
    else maxabs_rows<1>(a, s, k, row0, best);
    __syncthreads();
    for (int c = threadIdx.x; c < r0; c += blockDim.x)
      atomicMax(&a.keys[((size_t)s * a.K + k) * r0 + c], best[c]);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned total = gridDim.x * gridDim.y * gridDim.z;
    last = atomicAdd(a.ticket, 1u) == total - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // every other CTA's maxima are in place: the sign of each column's largest
  // entry, eight keys and then eight values in flight per thread
  const int n = 2 * a.K * r0;
  for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
    unsigned long long key[8];
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      key[u] = i < n ? __ldcg(a.keys + i) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      x[u] = 0.f;
      if (i < n) {
        const int si = i / (a.K * r0), ki = (i % (a.K * r0)) / r0, c = i % r0;
        const long long row = (long long)(0xffffffffu - (unsigned)(key[u] & 0xffffffffull));
        x[u] = __ldcg(a.f[si] + ((size_t)ki * a.d[si] + row) * r0 + c);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < n) a.sign[i] = x[u] < 0.f ? -1.f : 1.f;
    }
  }
}

// ------------------------------------------------------------ Gram pass
// grid (kPlMaxCtas, 2).  Each CTA stages tiles of L flattened elements of every
// expert (sign applied, fp64; L = a power of two with 4S * L <= kPlTileVals,
// S = ceil(K / 4)) and accumulates E E^T.  Thread tile (ti, tj), ti <= tj, owns
// the outputs (ti + S a, tj + S b), a, b < 4, and writes their transposes too
// (E E^T is symmetric: the tiles with ti > tj would repeat them).  The threads
// of a warp read consecutive tile entries (no bank conflicts).  Several thread
// groups split each tile's elements.  The next tile's values are loaded into
// registers while the current one is multiplied.
constexpr int kPlTileVals = 4096;                                      // values per staged tile
constexpr int kPlLoads = (kPlTileVals + kPlThreads - 1) / kPlThreads;  // per thread

// log2 of the staged tile length L for K experts
__host__ __device__ inline int pl_tile_shift(int K) {
  const int kp = 4 * ((K + 3) / 4);
  int l = 0;
  while ((2 << l) * kp <= kPlTileVals && (2 << l) <= 1024) ++l;
  return l;
}

struct GramSmem {
  union {
    double tile[kPlTileVals + 1024];   // [L][4S + 1]
    double red[kPlThreads][16];
  };
  int col[1024];                       // factor column of each element of the tile
};

template <int SC>   // SC = ceil(K / 4) known at compile time (offsets become immediates), 0 = runtime
__global__ void __launch_bounds__(kPlThreads, 2) pl_gram_kernel(PlaceArgs a) {
  const int s = blockIdx.y;
  if ((int)blockIdx.x >= a.ctas[s]) return;
  __shared__ GramSmem sm;
  const int K = a.K, r0 = a.r0;
  const long long D = a.d[s] * r0;   // flattened elements per expert
  const float *f = a.f[s];
  const float *sg = a.sign + (size_t)s * K * r0;
  const int S = SC ? SC : (K + 3) / 4;
  const int kp = 4 * S, ld = kp + 1;   // tile rows read (zero beyond K), row stride
  const int lshift = pl_tile_shift(4 * S);
  const int L = 1 << lshift;
  const int nt = S * (S + 1) / 2;      // upper-triangle thread tiles
  const int groups = kPlThreads / nt;
  const int t = threadIdx.x;
  const int tile_id = t % nt, grp = t / nt;
  const bool active = grp < groups;
  int ti = 0, rest = tile_id;
  while (rest >= S - ti) { rest -= S - ti; ++ti; }
  const int tj = ti + rest;
  double acc[4][4] = {};
  const long long nchunks = (D + L - 1) / L;
  float v[kPlLoads];
  auto load = [&](long long ch) {
    const long long f0 = ch * L;
#pragma unroll
    for (int u = 0; u < kPlLoads; ++u) {
      const int idx = t + u * kPlThreads;
      const int k = idx >> lshift, e = idx & (L - 1);
      v[u] = (k < K && f0 + e < D) ? __ldg(f + (size_t)k * D + f0 + e) : 0.f;
    }
  };
  long long ch = blockIdx.x;
  if (ch < nchunks) load(ch);
  for (; ch < nchunks; ch += a.ctas[s]) {
    __syncthreads();   // the previous tile is no longer read
    for (int e = t; e < L; e += kPlThreads) sm.col[e] = (int)((ch * L + e) % r0);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPlLoads; ++u) {
      const int idx = t + u * kPlThreads;
      const int k = idx >> lshift, e = idx & (L - 1);
      if (k < kp) sm.tile[e * ld + k] = k < K ? (double)(v[u] * __ldg(sg + k * r0 + sm.col[e])) : 0.0;
    }
    __syncthreads();
    if (ch + a.ctas[s] < nchunks) load(ch + a.ctas[s]);
    if (active) {
#pragma unroll 4
      for (int e = grp; e < L; e += groups) {
        const double *row = sm.tile + e * ld;
        double av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          av[i] = row[ti + S * i];
          bv[i] = row[tj + S * i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) sm.red[t][i * 4 + j] = acc[i][j];
  __syncthreads();
  double *out = a.part + ((size_t)s * kPlMaxCtas + blockIdx.x) * K * K;
  for (int o = t; o < nt * 16; o += kPlThreads) {
    const int tid = o / 16, ij = o % 16;
    int oi = 0, orest = tid;
    while (orest >= S - oi) { orest -= S - oi; ++oi; }
    const int oj = oi + orest;
    const int row = oi + S * (ij / 4), col = oj + S * (ij % 4);
    if (row >= K || col >= K) continue;
    double sum = 0.0;
    for (int g = 0; g < groups; ++g) sum += sm.red[g * nt + tid][ij];
    out[row * K + col] = sum;
    out[col * K + row] = sum;
  }
}

// The partials summed in a fixed order: a CTA sums 32 consecutive outputs,
// warp w the partials w, w + 16, ... (coalesced, several loads in flight), and
// the sixteen warps' sums are added in warp order.
constexpr int kPlSumWarps = 16;

__global__ void __launch_bounds__(32 * kPlSumWarps) pl_gram_sum_kernel(PlaceArgs a) {
  __shared__ double red[kPlSumWarps][32];
  const int kk = a.K * a.K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 32 + lane;   // over [2][K][K]
  const bool live = i < 2 * kk;
  const int s = live ? i / kk : 0, o = live ? i % kk : 0;
  const double *p = a.part + (size_t)s * kPlMaxCtas * kk + o;
  const int n = a.ctas[s];
  double sum = 0.0;
  if (live) {
#pragma unroll 4
    for (int c = warp; c < n; c += kPlSumWarps) sum += p[(size_t)c * kk];
  }
  red[warp][lane] = sum;
  __syncthreads();
  if (warp == 0 && live) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kPlSumWarps; ++w) t += red[w][lane];
    a.gram[i] = t;
  }
}

// ------------------------------------------------------------ K-Means
struct ClusterSmem {
  double g[kMaxExperts][kMaxExperts + 1];      // normalised Gram
  double alpha[kMaxExperts][kMaxExperts + 1];  // centre j = sum_i alpha[j][i] e_i
  double h[kMaxExperts][kMaxExperts + 1];      // (G alpha_j)_i
  double q[kMaxExperts];                       // alpha_j^T G alpha_j
  double nrm[kMaxExperts];                     // 1 / |e_i|
  double mind[kMaxExperts];
  int label[kMaxExperts];
  int count[kMaxExperts];
  int pick;
  int changed;
};

// Index of the largest (ties -> lowest index) of v[0..n) over one warp.
__device__ int warp_argmax(const double *v, int n) {
  const int lane = threadIdx.x & 31;
  double bv = -1.0;
  int bi = 0x7fffffff;
  for (int i = lane; i < n; i += 32)
    if (v[i] > bv) { bv = v[i]; bi = i; }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  return bi;
}

__global__ void __launch_bounds__(kPlClusterThreads) pl_cluster_kernel(PlaceArgs a) {
  extern __shared__ __align__(16) unsigned char pl_smem[];
  ClusterSmem &sm = *reinterpret_cast<ClusterSmem *>(pl_smem);
  const int s = blockIdx.x, K = a.K, t = threadIdx.x;
  const int C = (s == 0 ? a.M : a.N) < K ? (s == 0 ? a.M : a.N) : K;
  const double *G = a.gram + (size_t)s * K * K;
  for (int i = t; i < K; i += blockDim.x) {   // 1 / |e_i| (0 for a zero factor)
    const double v = G[i * K + i];
    sm.nrm[i] = v > 0.0 ? 1.0 / sqrt(v) : 0.0;
  }
  __syncthreads();
#pragma unroll 8
  for (int o = t; o < K * K; o += blockDim.x) {
    const int i = o / K, j = o % K;
    sm.g[i][j] = G[o] * sm.nrm[i] * sm.nrm[j];
  }
  for (int o = t; o < C * K; o += blockDim.x) sm.alpha[o / K][o % K] = 0.0;
  __syncthreads();
  // farthest-first traversal: centre 0 = expert 0, then the farthest expert
  if (t < 32) {
    int p = 0;
    for (int j = 0; j < C; ++j) {
      if (j > 0) p = warp_argmax(sm.mind, K);
      if (t == 0) sm.alpha[j][p] = 1.0;
      __syncwarp();
      for (int i = t; i < K; i += 32) {
        const double dij = sm.g[i][i] - 2.0 * sm.g[i][p] + sm.g[p][p];
        sm.mind[i] = (j == 0 || dij < sm.mind[i]) ? dij : sm.mind[i];
      }
      __syncwarp();
    }
  }
  __syncthreads();
  int it = 0;
  for (int pass = 0;; ++pass) {
    // distances from the centres' weights: h = G alpha_j, q_j = alpha_j . h_j
    for (int o = t; o < C * K; o += blockDim.x) {
      const int j = o / K, i = o % K;
      double acc[4] = {0.0, 0.0, 0.0, 0.0};   // four independent chains
      int l = 0;
      for (; l + 4 <= K; l += 4)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = fma(sm.alpha[j][l + u], sm.g[l + u][i], acc[u]);
      for (; l < K; ++l) acc[0] = fma(sm.alpha[j][l], sm.g[l][i], acc[0]);
      sm.h[j][i] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
    for (int j = t >> 5; j < C; j += blockDim.x >> 5) {   // one warp per centre
      const int lane = t & 31;
      double acc = 0.0;
      for (int i = lane; i < K; i += 32) acc = fma(sm.alpha[j][i], sm.h[j][i], acc);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) sm.q[j] = acc;
    }
    if (t == 0) sm.changed = 0;
    __syncthreads();
    for (int i = t; i < K; i += blockDim.x) {
      int best = 0;
      double bd = 0.0;
      for (int j = 0; j < C; ++j) {
        const double dij = sm.g[i][i] - 2.0 * sm.h[j][i] + sm.q[j];
        if (j == 0 || dij < bd) { bd = dij; best = j; }
      }
      if (pass == 0 || best != sm.label[i]) sm.changed = 1;
      sm.label[i] = best;
    }
    __syncthreads();
    if ((pass > 0 && !sm.changed) || it >= a.max_iter) break;
    // update: every centre with experts becomes their mean
    for (int j = t; j < C; j += blockDim.x) {
      int n = 0;
      for (int i = 0; i < K; ++i) n += sm.label[i] == j;
      sm.count[j] = n;
    }
    __syncthreads();
    for (int o = t; o < C * K; o += blockDim.x) {
      const int j = o / K, i = o % K;
      if (sm.count[j] > 0) sm.alpha[j][i] = sm.label[i] == j ? 1.0 / sm.count[j] : 0.0;
    }
    ++it;
    __syncthreads();
  }
  for (int i = t; i < K; i += blockDim.x) a.labels[s * K + i] = sm.label[i];
  if (t == 0) a.iters[s] = it;
}

// ------------------------------------------------------------ greedy placement
// key = distance << 32 | expert << 16 | cell: the smallest key is the next
// pair of the global greedy order.  Two warps; lane l of warp w holds expert
// 32 w + l's smallest key over the free cells.  Placing a cell invalidates only
// the experts whose best it was; the keys are double-buffered so that one
// barrier per round suffices.
__global__ void __launch_bounds__(kPlGreedyThreads) pl_greedy_kernel(PlaceArgs a) {
  __shared__ unsigned long long best[2][kMaxExperts];
  __shared__ unsigned char used[kMaxExperts * kMaxExperts];
  __shared__ int lab[2][kMaxExperts];
  const int K = a.K, M = a.M, N = a.N, cells = M * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long kNone = ~0ull;
  for (int c = threadIdx.x; c < cells; c += blockDim.x) used[c] = 0;
  for (int i = threadIdx.x; i < 2 * K; i += blockDim.x) lab[i / K][i % K] = a.labels[i];
  __syncthreads();
  auto best_of = [&](int k) {   // one warp: expert k's smallest key over the free cells
    const int mi = lab[0][k], ni = lab[1][k];
    unsigned long long b = kNone;
    for (int c = lane; c < cells; c += 32) {
      if (used[c]) continue;
      const int dm = c / N - mi, dn = c % N - ni;
      const unsigned long long key =
          ((unsigned long long)(dm * dm + dn * dn) << 32) | ((unsigned long long)k << 16) | (unsigned)c;
      b = key < b ? key : b;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, b, off);
      b = o < b ? o : b;
    }
    return b;
  };
  const int mine = warp * 32 + lane;   // this lane's expert
  // The distance-0 pairs come first in the greedy order, by expert index: an
  // expert takes its ideal cell unless a lower-index expert wants the same one.
  bool placed = false;
  if (mine < K) {
    const int ci = lab[0][mine] * N + lab[1][mine];
    bool first = true;
    for (int j = 0; j < mine && first; ++j) first = lab[0][j] * N + lab[1][j] != ci;
    if (first) {
      a.grid_assign[mine] = ci;
      used[ci] = 1;
      placed = true;
    }
  }
  const int remaining = K - __syncthreads_count(placed);
  const unsigned todo = __ballot_sync(0xffffffffu, mine < K && !placed);
  for (int l = 0; l < 32; ++l) {
    const int k = warp * 32 + l;
    if (k >= K) break;
    if (!(todo >> l & 1u)) {
      if (lane == l) best[0][k] = kNone;
      continue;
    }
    const unsigned long long b = best_of(k);
    if (lane == l) best[0][k] = b;
  }
  __syncthreads();
  for (int round = 0; round < remaining; ++round) {
    const int cur = round & 1, nxt = cur ^ 1;
    unsigned long long b = kNone;
    for (int k = lane; k < K; k += 32) b = best[cur][k] < b ? best[cur][k] : b;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, b, off);
      b = o < b ? o : b;
    }
    // K <= M*N leaves a free cell for every unplaced expert, so b is a real key
    const int ks = (int)((b >> 16) & 0xffff), cs = (int)(b & 0xffff);
    const bool ok = b != kNone && ks < K && cs < cells;
    if (ok && threadIdx.x == 0) a.grid_assign[ks] = cs;
    if (ok && lane == 0) used[cs] = 1;
    __syncwarp();
    unsigned long long key = mine < K ? best[cur][mine] : kNone;
    const bool redo = ok && mine < K && mine != ks && key != kNone && (int)(key & 0xffff) == cs;
    if (mine == ks) key = kNone;   // placed
    for (unsigned m = __ballot_sync(0xffffffffu, redo); m; m &= m - 1) {
      const int l = __ffs(m) - 1;
      const unsigned long long nb = best_of(warp * 32 + l);
      if (lane == l) key = nb;
    }
    if (mine < K) best[nxt][mine] = key;
    __syncthreads();
  }
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    if (a.ideal) {
      a.ideal[2 * k] = lab[0][k];
      a.ideal[2 * k + 1] = lab[1][k];
    }
  }
  if (threadIdx.x < 2 && a.iterations) a.iterations[threadIdx.x] = a.iters[threadIdx.x];
}

// ------------------------------------------------------------ host side
struct PlaceWs {
  size_t keys, ticket, sign, part, gram, labels, iters, total;
};

size_t pl_align(size_t x) { return (x + 255) / 256 * 256; }

PlaceWs place_ws(int K, int r0) {
  PlaceWs w{};
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += pl_align(b);
    return o;
  };
  w.keys = take((size_t)2 * K * r0 * 8);
  w.ticket = take(4);   // directly after keys: one memset clears both
  w.sign = take((size_t)2 * K * r0 * 4);
  w.part = take((size_t)2 * kPlMaxCtas * K * K * 8);
  w.gram = take((size_t)2 * K * K * 8);
  w.labels = take((size_t)2 * K * 4);
  w.iters = take(2 * 4);
  w.total = off;
  return w;
}

tileq_status place_check(const tileq_place_in *in) {
  if (!in) return TILEQ_ERR_INVALID_ARG;
  if (in->K < 1 || in->M < 1 || in->N < 1 || in->d_u < 1 || in->d_v < 1 || in->r0 < 1)
    return TILEQ_ERR_INVALID_ARG;
  if (in->K > kMaxExperts || in->M > kMaxExperts || in->N > kMaxExperts || in->r0 > kPlMaxR0)
    return TILEQ_ERR_UNSUPPORTED;
  if ((long long)in->M * in->N < in->K) return TILEQ_ERR_INVALID_ARG;
  if (in->max_iter < 1) return TILEQ_ERR_INVALID_ARG;
  if (in->max_iter > TILEQ_PLACE_MAX_ITER) return TILEQ_ERR_UNSUPPORTED;
  return TILEQ_OK;
}

}  // namespace
}  // namespace tileq

using namespace tileq;

extern "C" tileq_status tileq_place_workspace_size(const tileq_place_in *in, size_t *bytes) {
  if (!bytes) return TILEQ_ERR_INVALID_ARG;
  const tileq_status st = place_check(in);
  if (st != TILEQ_OK) return st;
  *bytes = place_ws(in->K, in->r0).total;
  return TILEQ_OK;
}

extern "C" tileq_status tileq_place_experts(const tileq_place_in *in, tileq_place_out *out, void *ws,
                                            size_t ws_bytes, tileq_stream_t stream_) {
  const tileq_status st = place_check(in);
  if (st != TILEQ_OK) return st;
  if (!in->u || !in->v || !out || !out->grid_assign || !ws) return TILEQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(in->u) % 16 || reinterpret_cast<uintptr_t>(in->v) % 16 ||
      reinterpret_cast<uintptr_t>(ws) % 16)
    return TILEQ_ERR_INVALID_ARG;
  const PlaceWs w = place_ws(in->K, in->r0);
  if (ws_bytes < w.total) return TILEQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  char *base = static_cast<char *>(ws);
  PlaceArgs a;
  a.f[0] = in->u;
  a.f[1] = in->v;
  a.d[0] = in->d_u;
  a.d[1] = in->d_v;
  a.K = in->K;
  a.M = in->M;
  a.N = in->N;
  a.r0 = in->r0;
  a.max_iter = in->max_iter;
  for (int side = 0; side < 2; ++side) {
    const long long L = 1LL << pl_tile_shift(a.K);
    const long long nchunks = (a.d[side] * a.r0 + L - 1) / L;
    const long long want = (nchunks + kPlMinChunks - 1) / kPlMinChunks;
    a.ctas[side] = (int)std::max(1LL, std::min<long long>(want, kPlMaxCtas));
  }
  a.keys = reinterpret_cast<unsigned long long *>(base + w.keys);
  a.ticket = reinterpret_cast<unsigned *>(base + w.ticket);
  a.sign = reinterpret_cast<float *>(base + w.sign);
  a.part = reinterpret_cast<double *>(base + w.part);
  a.gram = reinterpret_cast<double *>(base + w.gram);
  a.labels = reinterpret_cast<int32_t *>(base + w.labels);
  a.iters = reinterpret_cast<int32_t *>(base + w.iters);
  a.grid_assign = out->grid_assign;
  a.ideal = out->ideal;
  a.iterations = out->iterations;

#define PL(call)                                      \
  do {                                                \
    if ((call) != cudaSuccess) return TILEQ_ERR_CUDA; \
  } while (0)
  mark_stage(0, s);
  PL(cudaMemsetAsync(base + w.keys, 0, w.ticket + 4 - w.keys, s));
  const long long dmax = std::max(a.d[0], a.d[1]);
  const unsigned row_chunks = (unsigned)((dmax + kPlRowsPerCta - 1) / kPlRowsPerCta);
  const int mthreads = std::max(32, (256 / a.r0) * a.r0);
  pl_maxabs_kernel<<<dim3(row_chunks, a.K, 2), mthreads, 0, s>>>(a);
  mark_stage(1, s);
  const dim3 ggrid(kPlMaxCtas, 2);
  switch ((a.K + 3) / 4) {   // the layer shapes' expert counts get compile-time tile strides
    case 16: pl_gram_kernel<16><<<ggrid, kPlThreads, 0, s>>>(a); break;
    case 15: pl_gram_kernel<15><<<ggrid, kPlThreads, 0, s>>>(a); break;
    case 2: pl_gram_kernel<2><<<ggrid, kPlThreads, 0, s>>>(a); break;
    default: pl_gram_kernel<0><<<ggrid, kPlThreads, 0, s>>>(a);
  }
  mark_stage(2, s);
  pl_gram_sum_kernel<<<(2 * a.K * a.K + 31) / 32, 32 * kPlSumWarps, 0, s>>>(a);
  const size_t csmem = sizeof(ClusterSmem);
  PL(cudaFuncSetAttribute(pl_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem));
  pl_cluster_kernel<<<2, kPlClusterThreads, csmem, s>>>(a);
  mark_stage(3, s);
  pl_greedy_kernel<<<1, kPlGreedyThreads, 0, s>>>(a);
  mark_stage(4, s);
  count_launches(5);
  PL(cudaGetLastError());
#undef PL
  return TILEQ_OK;
}
