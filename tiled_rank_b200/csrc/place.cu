// Expert placement on the M x N tile grid: TileQ summary, section 2.1, steps
// 2-4 (feature embeddings from each expert's rank-r0 SVD factors, a K-Means
// biclustering that gives every expert an ideal grid coordinate, and a greedy
// spatial allocation that resolves experts wanting the same tile).
//
//   pl_maxabs_kernel     per factor column, the entry of largest magnitude
//                        (64-bit atomicMax on |x| bits : ~row, so ties keep the
//                        first row)
//   pl_sign_kernel       the column's sign from that entry
//   pl_gram_kernel       partial fp64 Gram matrices E E^T of the sign-fixed,
//                        flattened factors, one per CTA over its slice of the
//                        flattened dimension (both sides in one launch)
//   pl_gram_sum_kernel   the partials summed in a fixed order (deterministic)
//   pl_cluster_kernel    one CTA per side: normalisation (folded into the Gram:
//                        G_ij / (|e_i| |e_j|)), farthest-first start, Lloyd
//                        iterations with every centre held as weights over the
//                        experts, so that |e_i - c_j|^2 = G_ii - 2 (G a_j)_i + a_j^T G a_j
//   pl_greedy_kernel     one CTA: the global greedy allocation, each round
//                        placing the smallest (distance, expert, cell) key over
//                        the experts' cached best free cells
//
// The factors are read twice (the sign pass and the Gram pass); everything
// after the Gram works on K x K numbers.
#include "kernels.cuh"

namespace tileq {
namespace {

constexpr int kPlMaxR0 = TILEQ_PLACE_MAX_R0;
constexpr int kPlChunk = 64;        // flattened elements per Gram tile
constexpr int kPlThreads = 256;     // Gram CTA: 16 x 16 threads of 4 x 4 outputs at K = 64
constexpr int kPlMaxCtas = 148;     // Gram CTAs per side (partials summed afterwards)
constexpr int kPlMinChunks = 8;     // at least this many tiles per Gram CTA
constexpr int kPlRowsPerCta = 64;   // factor rows per CTA of the sign pass
constexpr int kPlClusterThreads = 1024;
constexpr int kPlGreedyThreads = 1024;

struct PlaceArgs {
  const float *f[2];          // U side, V side: [K][d][r0]
  long long d[2];             // rows of each side's factors
  int K, M, N, r0, max_iter;
  int ctas[2];                // Gram CTAs per side
  unsigned long long *keys;   // [2][K][r0]
  float *sign;                // [2][K][r0]
  double *part;               // [2][kPlMaxCtas][K][K]
  double *gram;               // [2][K][K]
  int32_t *labels;            // [2][K]
  int32_t *iters;             // [2]
  int32_t *grid_assign, *ideal, *iterations;
};

// ------------------------------------------------------------ sign pass
// grid (row chunks, K, 2 sides); thread t handles column t % r0 of rows
// t / r0, t / r0 + rows_per_step, ... of its chunk.
__global__ void __launch_bounds__(256) pl_maxabs_kernel(PlaceArgs a) {
  const int s = blockIdx.z, k = blockIdx.y;
  const long long d = a.d[s];
  const long long row0 = (long long)blockIdx.x * kPlRowsPerCta;
  if (row0 >= d) return;
  const int r0 = a.r0;
  const int lanes = (blockDim.x / r0) * r0;   // threads in use: whole rows
  __shared__ unsigned long long best[kPlMaxR0];
  for (int c = threadIdx.x; c < r0; c += blockDim.x) best[c] = 0ull;
  __syncthreads();
  if (threadIdx.x < lanes) {
    const int c = threadIdx.x % r0;
    const int step = lanes / r0;
    const long long row_end = row0 + kPlRowsPerCta < d ? row0 + kPlRowsPerCta : d;
    const float *f = a.f[s] + (size_t)k * d * r0;
    unsigned long long key = 0ull;
    for (long long row = row0 + threadIdx.x / r0; row < row_end; row += step) {
      const float x = f[row * r0 + c];
      const unsigned long long kx =
          ((unsigned long long)(__float_as_uint(x) & 0x7fffffffu) << 32) | (0xffffffffu - (unsigned)row);
      key = kx > key ? kx : key;
    }
    atomicMax(&best[c], key);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < r0; c += blockDim.x)
    atomicMax(&a.keys[((size_t)s * a.K + k) * r0 + c], best[c]);
}

__global__ void pl_sign_kernel(PlaceArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;   // over [2][K][r0]
  const int per_side = a.K * a.r0;
  if (i >= 2 * per_side) return;
  const int s = i / per_side, k = (i % per_side) / a.r0, c = i % a.r0;
  const unsigned long long key = a.keys[i];
  const long long row = (long long)(0xffffffffu - (unsigned)(key & 0xffffffffull));
  const float x = a.f[s][((size_t)k * a.d[s] + row) * a.r0 + c];
  a.sign[i] = x < 0.f ? -1.f : 1.f;
}

// ------------------------------------------------------------ Gram pass
// grid (kPlMaxCtas, 2).  Each CTA stages tiles of kPlChunk flattened elements
// of every expert (sign applied, fp64) and accumulates 4 x 4 blocks of E E^T;
// below K = 64 several thread groups split each tile's elements.
struct GramSmem {
  union {
    double tile[kPlChunk][kMaxExperts + 1];
    double red[kPlThreads][16];
  };
};

__global__ void __launch_bounds__(kPlThreads) pl_gram_kernel(PlaceArgs a) {
  const int s = blockIdx.y;
  if ((int)blockIdx.x >= a.ctas[s]) return;
  __shared__ GramSmem sm;
  const int K = a.K, r0 = a.r0;
  const long long D = a.d[s] * r0;   // flattened elements per expert
  const float *f = a.f[s];
  const float *sg = a.sign + (size_t)s * K * r0;
  const int nt1 = (K + 3) / 4, nt = nt1 * nt1;
  const int groups = kPlThreads / nt;
  const int t = threadIdx.x;
  const int tile_id = t % nt, grp = t / nt;
  const int ti = tile_id / nt1, tj = tile_id % nt1;
  const bool active = grp < groups;
  const int kp = nt1 * 4;            // rows of the tile that the blocks read (zero beyond K)
  double acc[4][4] = {};
  const long long nchunks = (D + kPlChunk - 1) / kPlChunk;
  for (long long ch = blockIdx.x; ch < nchunks; ch += a.ctas[s]) {
    const long long f0 = ch * kPlChunk;
    __syncthreads();
    for (int idx = t; idx < kp * kPlChunk; idx += kPlThreads) {
      const int k = idx / kPlChunk, e = idx % kPlChunk;
      double x = 0.0;
      if (k < K && f0 + e < D) {
        const long long fi = f0 + e;
        x = (double)(f[(size_t)k * D + fi] * sg[k * r0 + (int)(fi % r0)]);
      }
      sm.tile[e][k] = x;
    }
    __syncthreads();
    if (active) {
      for (int e = grp; e < kPlChunk; e += groups) {
        double av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          av[i] = sm.tile[e][4 * ti + i];
          bv[i] = sm.tile[e][4 * tj + i];
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
    const int row = 4 * (tid / nt1) + ij / 4, col = 4 * (tid % nt1) + ij % 4;
    if (row >= K || col >= K) continue;
    double sum = 0.0;
    for (int g = 0; g < groups; ++g) sum += sm.red[g * nt + tid][ij];
    out[row * K + col] = sum;
  }
}

__global__ void pl_gram_sum_kernel(PlaceArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;   // over [2][K][K]
  const int kk = a.K * a.K;
  if (i >= 2 * kk) return;
  const int s = i / kk, o = i % kk;
  const double *p = a.part + (size_t)s * kPlMaxCtas * kk + o;
  double sum = 0.0;
  for (int c = 0; c < a.ctas[s]; ++c) sum += p[(size_t)c * kk];
  a.gram[i] = sum;
}

// ------------------------------------------------------------ K-Means
struct ClusterSmem {
  double g[kMaxExperts][kMaxExperts + 1];      // normalised Gram
  double alpha[kMaxExperts][kMaxExperts + 1];  // centre j = sum_i alpha[j][i] e_i
  double h[kMaxExperts][kMaxExperts + 1];      // (G alpha_j)_i
  double q[kMaxExperts];                       // alpha_j^T G alpha_j
  double nrm[kMaxExperts];
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
  for (int i = t; i < K; i += blockDim.x) {
    const double v = G[i * K + i];
    sm.nrm[i] = v > 0.0 ? sqrt(v) : 0.0;
  }
  __syncthreads();
  for (int o = t; o < K * K; o += blockDim.x) {
    const int i = o / K, j = o % K;
    sm.g[i][j] = (sm.nrm[i] > 0.0 && sm.nrm[j] > 0.0) ? G[o] / sm.nrm[i] / sm.nrm[j] : 0.0;
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
      double acc = 0.0;
      for (int l = 0; l < K; ++l) acc = fma(sm.alpha[j][l], sm.g[l][i], acc);
      sm.h[j][i] = acc;
    }
    __syncthreads();
    if (t < 32) {
      for (int j = 0; j < C; ++j) {
        double acc = 0.0;
        for (int i = t; i < K; i += 32) acc = fma(sm.alpha[j][i], sm.h[j][i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (t == 0) sm.q[j] = acc;
      }
      if (t == 0) sm.changed = 0;
    }
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
// pair of the global greedy order.  best[k] caches expert k's smallest key over
// the free cells; placing a cell invalidates only the experts whose best it was.
__global__ void __launch_bounds__(kPlGreedyThreads) pl_greedy_kernel(PlaceArgs a) {
  __shared__ unsigned long long best[kMaxExperts];
  __shared__ unsigned char used[kMaxExperts * kMaxExperts];
  __shared__ int placed_cell;
  const int K = a.K, M = a.M, N = a.N, cells = M * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const unsigned long long kNone = ~0ull;
  for (int c = threadIdx.x; c < cells; c += blockDim.x) used[c] = 0;
  __syncthreads();
  auto best_of = [&](int k) {   // one warp: expert k's smallest key over the free cells
    const int mi = a.labels[k], ni = a.labels[K + k];
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
  for (int k = warp; k < K; k += nwarps) {
    const unsigned long long b = best_of(k);
    if (lane == 0) best[k] = b;
  }
  __syncthreads();
  for (int round = 0; round < K; ++round) {
    if (warp == 0) {
      unsigned long long b = kNone;
      for (int k = lane; k < K; k += 32) b = best[k] < b ? best[k] : b;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, b, off);
        b = o < b ? o : b;
      }
      if (lane == 0) {
        // K <= M*N leaves a free cell for every unplaced expert, so b is a real key
        const int k = (int)((b >> 16) & 0xffff), c = (int)(b & 0xffff);
        if (b != kNone && k < K && c < cells) {
          a.grid_assign[k] = c;
          used[c] = 1;
          best[k] = kNone;   // placed
        }
        placed_cell = c;
      }
    }
    __syncthreads();
    const int c = placed_cell;
    for (int k = warp; k < K; k += nwarps) {
      if (best[k] == kNone || (int)(best[k] & 0xffff) != c) continue;
      const unsigned long long b = best_of(k);
      if (lane == 0) best[k] = b;
    }
    __syncthreads();
  }
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    if (a.ideal) {
      a.ideal[2 * k] = a.labels[k];
      a.ideal[2 * k + 1] = a.labels[K + k];
    }
  }
  if (threadIdx.x < 2 && a.iterations) a.iterations[threadIdx.x] = a.iters[threadIdx.x];
}

// ------------------------------------------------------------ host side
struct PlaceWs {
  size_t keys, sign, part, gram, labels, iters, total;
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
    const long long nchunks = (a.d[side] * a.r0 + kPlChunk - 1) / kPlChunk;
    const long long want = (nchunks + kPlMinChunks - 1) / kPlMinChunks;
    a.ctas[side] = (int)std::max(1LL, std::min<long long>(want, kPlMaxCtas));
  }
  a.keys = reinterpret_cast<unsigned long long *>(base + w.keys);
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
  PL(cudaMemsetAsync(a.keys, 0, (size_t)2 * a.K * a.r0 * 8, s));
  const long long dmax = std::max(a.d[0], a.d[1]);
  const unsigned row_chunks = (unsigned)((dmax + kPlRowsPerCta - 1) / kPlRowsPerCta);
  const int mthreads = std::max(32, (256 / a.r0) * a.r0);
  pl_maxabs_kernel<<<dim3(row_chunks, a.K, 2), mthreads, 0, s>>>(a);
  pl_sign_kernel<<<(2 * a.K * a.r0 + 255) / 256, 256, 0, s>>>(a);
  pl_gram_kernel<<<dim3(kPlMaxCtas, 2), kPlThreads, 0, s>>>(a);
  pl_gram_sum_kernel<<<(2 * a.K * a.K + 255) / 256, 256, 0, s>>>(a);
  const size_t csmem = sizeof(ClusterSmem);
  PL(cudaFuncSetAttribute(pl_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem));
  pl_cluster_kernel<<<2, kPlClusterThreads, csmem, s>>>(a);
  pl_greedy_kernel<<<1, kPlGreedyThreads, 0, s>>>(a);
  count_launches(6);
  PL(cudaGetLastError());
#undef PL
  return TILEQ_OK;
}
