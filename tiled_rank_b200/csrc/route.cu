// Routing and permutation kernels of the TileQ MoE forward.
//
// route_kernel    : one warp per token: exact top-k of the fp32 logits (descending,
//                   equal logits -> lower expert id), softmax over the chosen
//                   logits (or, full_softmax, their entries of the softmax over
//                   all K logits), and the bf16 -> fp16 conversion of x.
// route_permute_kernel: up to 4096 pairs, routing and, in CTA 0, the
//                   deterministic stable counting sort of the (token, slot)
//                   pairs by expert and the GEMM tile tables; per slot, the
//                   row of the projected [T, N, r] tensor it reads (TileQ
//                   paper, section 2.2) and, for the linear layer, whether it
//                   is the token's first slot in its grid row (the in-place
//                   accumulation).
// permute_count_kernel + permute_scatter_kernel: the same sort and tables for
//                   long batches, one CTA per 1024 pairs.
#include "kernels.cuh"

namespace tileq {

// Zero the split-K arrival counters and copy x from bf16 to fp16; thread tid
// of nthreads, four 16-byte chunks in flight per thread.
__device__ __forceinline__ void zero_and_convert(const RouteArgs &a, long long tid, long long nthreads) {
  for (long long i = tid; i < a.nzero; i += nthreads) a.zero[i] = 0;
  if (a.x == nullptr) return;
  const long long nchunk = (long long)a.T * (a.d_x / 8);
  const uint4 *src = reinterpret_cast<const uint4 *>(a.x);
  uint4 *dst = reinterpret_cast<uint4 *>(a.x16);
  for (long long c0 = tid; c0 < nchunk; c0 += 4 * nthreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long c = c0 + u * nthreads;
      if (c < nchunk) v[u] = src[c];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long c = c0 + u * nthreads;
      if (c >= nchunk) continue;
      const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
      uint4 o;
      __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        h[i] = half2_checked(f.x, f.y, a.status);
      }
      dst[c] = o;
    }
  }
}

// Top-k and weights of token t by one warp.
__device__ __forceinline__ void route_token(const RouteArgs &a, int t, int lane) {
  const float NEG = -INFINITY;
  const float *lg = a.logits + (size_t)t * a.K;
  // a NaN logit ranks as -inf: every comparison below is then a total order,
  // so all lanes agree on the winners
  float v0 = lane < a.K ? lg[lane] : NEG;
  float v1 = lane + 32 < a.K ? lg[lane + 32] : NEG;
  if (isnan(v0)) v0 = NEG;
  if (isnan(v1)) v1 = NEG;
  bool used0 = lane >= a.K, used1 = lane + 32 >= a.K;
  float sel_v[kMaxTopK];
  int sel_i[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < a.k) {
      float bv = NEG;
      int bi = 0x7fffffff;
      if (!used0) { bv = v0; bi = lane; }
      if (!used1 && (used0 || v1 > v0)) { bv = v1; bi = lane + 32; }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (bi == lane) used0 = true;
      if (bi == lane + 32) used1 = true;
      sel_v[j] = bv;
      sel_i[j] = bi;
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < a.k) sum += expf(sel_v[j] - sel_v[0]);
  if (a.full_softmax) {
    // the denominator runs over every logit; sel_v[0] is the row maximum
    float s = (lane < a.K ? expf(v0 - sel_v[0]) : 0.f) + (lane + 32 < a.K ? expf(v1 - sel_v[0]) : 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    sum = s;
  }
  // every chosen logit -inf (or NaN): equal weights, the limit of equal logits
  const bool none = sel_v[0] == NEG;
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k) {
        a.topk_idx[t * a.k + j] = sel_i[j];
        a.topk_w[t * a.k + j] = none ? 1.0f / (a.full_softmax ? a.K : a.k) : expf(sel_v[j] - sel_v[0]) / sum;
      }
    }
  }
}

__global__ void __launch_bounds__(256) route_kernel(RouteArgs a) {
  pdl_wait_and_release();
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  zero_and_convert(a, gtid, (long long)gridDim.x * blockDim.x);
  const int warp = (int)(gtid >> 5);
  if (warp < a.T) route_token(a, warp, threadIdx.x & 31);
}

// ---------------------------------------------------------------------------
// single-CTA stable counting sort
// ---------------------------------------------------------------------------
constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;

struct SortSmem {
  int hist[kPermWarps][kMaxExperts];
  int total[kMaxExperts + 1];
};

// Sort the items 0..n-1 whose key(i) >= 0 by key, stably.  dest[i] receives the
// sorted position of a valid item; offsets[0..nkeys] the bucket starts.
template <typename KeyFn>
__device__ void cta_stable_sort(int n, int nkeys, KeyFn key, int *dest, int *offsets,
                                SortSmem &s) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kPermWarps * kMaxExperts; i += blockDim.x)
    (&s.hist[0][0])[i] = 0;
  __syncthreads();
  const int chunk = (n + kPermWarps - 1) / kPermWarps;
  const int c0 = min(n, warp * chunk), c1 = min(n, c0 + chunk);
  for (int i = c0 + lane; i < c1; i += 32) {
    const int kk = key(i);
    if (kk >= 0) atomicAdd(&s.hist[warp][kk], 1);
  }
  __syncthreads();
  if (threadIdx.x < nkeys) {
    int tot = 0;
    for (int w = 0; w < kPermWarps; ++w) tot += s.hist[w][threadIdx.x];
    s.total[threadIdx.x] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int kk = 0; kk < nkeys; ++kk) {
      const int tt = s.total[kk];
      s.total[kk] = run;
      offsets[kk] = run;
      run += tt;
    }
    offsets[nkeys] = run;
    s.total[nkeys] = run;
  }
  __syncthreads();
  if (threadIdx.x < nkeys) {
    int run = s.total[threadIdx.x];
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = s.hist[w][threadIdx.x];
      s.hist[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int base = c0; base < c1; base += 32) {
    const int i = base + lane;
    const int kk = i < c1 ? key(i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, kk);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (kk >= 0) pos = s.hist[warp][kk] + rank;
    __syncwarp();
    if (kk >= 0) {
      dest[i] = pos;
      if (rank == 0) s.hist[warp][kk] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
}

// Fill a tile table: group g owns items [off[g], off[g+1]) split into tiles of bn.
__device__ void build_tiles(const int *off, int ngroups, int bn, int4 *tiles, int *count,
                            int *first /* [ngroups+1] or null */,
                            int *scratch /* smem [kMaxExperts+1] */) {
  if (threadIdx.x < ngroups) {
    const int cnt = off[threadIdx.x + 1] - off[threadIdx.x];
    scratch[threadIdx.x] = (cnt + bn - 1) / bn;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int g = 0; g < ngroups; ++g) {
      const int c = scratch[g];
      scratch[g] = run;
      run += c;
    }
    scratch[ngroups] = run;
    *count = run;
  }
  __syncthreads();
  if (first != nullptr && threadIdx.x <= ngroups) first[threadIdx.x] = scratch[threadIdx.x];
  if (threadIdx.x < ngroups) {
    const int g = threadIdx.x;
    const int i0 = off[g], i1 = off[g + 1];
    int ti = scratch[g];
    for (int i = i0; i < i1; i += bn) tiles[ti++] = make_int4(g, i, min(bn, i1 - i), 0);
  }
  __syncthreads();
}

// The tables of one sorted pair p placed at slot: the pair itself, its token and
// weight; its row of the projected [T, N, r] tensor per z projection (TileQ
// paper, section 2.2: project once, select by routing); and for the in-place
// accumulation per (token, grid row), whether it is the token's first slot in
// its grid row (that slot carries a_{t,m}, the others carry zeros).
__device__ __forceinline__ void write_slot(const PermuteArgs &a, int p, int slot) {
  const int k = a.k;
  const int t = p / k, j = p - t * k;
  const int e = a.topk_idx[p];
  a.sorted_pairs[slot] = p;
  a.slot_of_pair[p] = slot;
  a.slot_tok[slot] = t;
  a.slot_w[slot] = a.topk_w[p];
  for (int zp = 0; zp < a.n_zproj; ++zp) a.zidx[zp][slot] = t * a.N + a.n_of[zp][e];
  if (a.row_proj >= 0) {
    const int8_t *mrow = a.m_of_row;
    const int r = mrow[e];
    bool designated = true;
    for (int jj = 0; jj < j; ++jj)
      if (mrow[a.topk_idx[t * k + jj]] == r) designated = false;
    a.aidx[slot] = designated ? 1 : -1;
  }
}

// Routing and the one-CTA permutation in one launch (batches of at most
// kPermMultiMin pairs): CTA 0 routes every token (one warp per token) and
// sorts the pairs; the other CTAs zero the counters and convert x.  The top-k
// results CTA 0 writes are visible to its own threads after the barrier.
__global__ void __launch_bounds__(kPermThreads) route_permute_kernel(RouteArgs ra, PermuteArgs a) {
  pdl_wait_and_release();
  if (blockIdx.x != 0 || gridDim.x == 1)
    zero_and_convert(ra, (long long)(blockIdx.x - (gridDim.x > 1)) * blockDim.x + threadIdx.x,
                     (long long)(gridDim.x - (gridDim.x > 1)) * blockDim.x);
  if (blockIdx.x != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < ra.T; t += kPermWarps) route_token(ra, t, lane);
  __syncthreads();
  __shared__ SortSmem s;
  __shared__ int scratch[kMaxExperts + 1];
  const int P = a.T * a.k;
  const int32_t *idx = a.topk_idx;
  cta_stable_sort(P, a.K, [&](int p) { return idx[p]; }, a.dest, a.expert_offsets, s);
  for (int p = threadIdx.x; p < P; p += blockDim.x) write_slot(a, p, a.dest[p]);
  __syncthreads();
  build_tiles(a.expert_offsets, a.K, a.bn, a.tiles_main, a.tile_counts + 0, a.tile_first_main, scratch);
  if (a.bn_wide > 0)
    build_tiles(a.expert_offsets, a.K, a.bn_wide, a.tiles_wide, a.tile_counts + 1, nullptr, scratch);
}

// ---------------------------------------------------------------------------
// multi-CTA stable counting sort for long batches: CTA c owns the pairs
// [c*kPermChunk, (c+1)*kPermChunk).  permute_count_kernel stores each CTA's
// per-expert counts; permute_scatter_kernel derives from them where the CTA's
// pairs of each expert start and places them in pair order, so the result is
// the same stable order as the one-CTA sort.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPermChunkThreads) permute_count_kernel(PermuteArgs a) {
  pdl_wait_and_release();
  __shared__ int hist[kMaxExperts];
  const int P = a.T * a.k;
  for (int e = threadIdx.x; e < a.K; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kPermChunk, p1 = min(P, p0 + kPermChunk);
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) atomicAdd(&hist[a.topk_idx[p]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < a.K; e += blockDim.x) a.pcounts[blockIdx.x * a.K + e] = hist[e];
}

__global__ void __launch_bounds__(kPermChunkThreads) permute_scatter_kernel(PermuteArgs a) {
  pdl_wait_and_release();
  constexpr int W = kPermChunkThreads / 32;
  constexpr int kParts = kPermChunkThreads / kMaxExperts;
  static_assert(kPermChunk % W == 0 && kParts >= 1, "chunk split");
  __shared__ int hist[W][kMaxExperts];
  __shared__ int red[2][kParts][kMaxExperts];
  __shared__ int before[kMaxExperts];
  __shared__ int start[kMaxExperts + 1];
  __shared__ int scratch[kMaxExperts + 1];
  const int P = a.T * a.k, K = a.K, C = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t *idx = a.topk_idx;

  // 1. per expert: pairs in all CTAs (the bucket sizes) and in the CTAs before this one
  {
    const int e = threadIdx.x % kMaxExperts, part = threadIdx.x / kMaxExperts;
    int b = 0, tot = 0;
    if (e < K) {
      for (int cc = part; cc < C; cc += kParts) {
        const int v = a.pcounts[cc * K + e];
        tot += v;
        if (cc < c) b += v;
      }
    }
    red[0][part][e] = b;
    red[1][part][e] = tot;
  }
  for (int i = threadIdx.x; i < W * kMaxExperts; i += blockDim.x) (&hist[0][0])[i] = 0;
  __syncthreads();
  if (threadIdx.x < K) {
    int b = 0, tot = 0;
    for (int q = 0; q < kParts; ++q) {
      b += red[0][q][threadIdx.x];
      tot += red[1][q][threadIdx.x];
    }
    before[threadIdx.x] = b;
    start[threadIdx.x] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < K; ++e) {
      const int n = start[e];
      start[e] = run;
      run += n;
    }
    start[K] = run;
  }
  __syncthreads();
  if (c == 0) {
    for (int e = threadIdx.x; e <= K; e += blockDim.x) a.expert_offsets[e] = start[e];
    build_tiles(start, K, a.bn, a.tiles_main, a.tile_counts + 0, a.tile_first_main, scratch);
    if (a.bn_wide > 0) build_tiles(start, K, a.bn_wide, a.tiles_wide, a.tile_counts + 1, nullptr, scratch);
  }

  // 2. this CTA's pairs, split into W contiguous runs, one per warp
  const int p0 = c * kPermChunk, p1 = min(P, p0 + kPermChunk);
  constexpr int sub = kPermChunk / W;
  const int w0 = min(p1, p0 + warp * sub), w1 = min(p1, w0 + sub);
  for (int i = w0 + lane; i < w1; i += 32) atomicAdd(&hist[warp][idx[i]], 1);
  __syncthreads();
  if (threadIdx.x < K) {
    int run = start[threadIdx.x] + before[threadIdx.x];
    for (int w = 0; w < W; ++w) {
      const int n = hist[w][threadIdx.x];
      hist[w][threadIdx.x] = run;
      run += n;
    }
  }
  __syncthreads();
  // 3. stable placement: equal experts within 32 pairs ranked by lane
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const int kk = i < w1 ? idx[i] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, kk);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int pos = kk >= 0 ? hist[warp][kk] + rank : 0;
    __syncwarp();
    if (kk >= 0) {
      write_slot(a, i, pos);
      if (rank == 0) hist[warp][kk] += __popc(peers);
    }
    __syncwarp();
  }
}

}  // namespace tileq
