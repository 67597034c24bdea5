// Kernel argument structs and launch entry points shared by the .cu files.
#pragma once
#include "common.cuh"

namespace tileq {

// ---------------------------------------------------------------- routing
struct RouteArgs {
  const float *logits;
  const __nv_bfloat16 *x;  // may be null (route only)
  __half *x16;
  int d_x, T, K, k;
  int32_t *topk_idx;
  float *topk_w;
};

struct PermuteArgs {
  int T, k, K, M, N, bn;
  const int32_t *topk_idx;
  const float *topk_w;
  int *dest;               // scratch [P]
  int32_t *expert_offsets; // [K+1]
  int32_t *sorted_pairs;   // [P]
  int *slot_of_pair;       // [P]
  int *slot_tok;           // [P]
  float *slot_w;           // [P]
  int4 *tiles_main;        // [P/bn + K]
  int *tile_first_main;    // [K+1] first tile of each expert
  int *tile_counts;        // [4]: main, z0, z1, rows
  int n_zproj;             // 0, 1 or 2
  int8_t n_of[2][kMaxExperts];
  int *col_offsets[2];     // [N+1]
  int *colpair_tok[2];     // [P]
  int *zidx[2];            // slot -> colpair
  int4 *tiles_z[2];        // [P/bn + N]
  int row_proj;            // -1 = no row sort
  int8_t m_of_row[kMaxExperts];
  int *row_offsets;        // [M+1]
  int *rowpair_tok;        // [P]
  int *rowpair_row;        // [P]
  int *aidx;               // slot -> rowpair (or -1 when not the designated pair)
};

// ---------------------------------------------------------------- GEMM
enum AMode { AM_Q2 = 0, AM_F16 = 1 };
enum Epi { EPI_SWIGLU_H = 0, EPI_STORE_F32 = 1, EPI_STORE_F16 = 2, EPI_ACCUM_F32 = 3,
           EPI_STORE2_F32 = 4 };

// One grouped GEMM  out[item][o] = sum_k A_g[o][k] * B[row(item)][k]  (+ low-rank
// extension), items grouped by tiles (group, item0, nitems).  A rows are
// output features; items are tokens / slots / (token, column) pairs.
struct GemmProblem {
  const int4 *tiles;
  const int *tile_count;
  int static_items;       // tiles == nullptr: one group 0 holding this many items
  int only_group;         // >= 0: tiles [group_first_tile[g], group_first_tile[g+1]) only
  const int *group_first_tile;
  int d_out, d_in;
  const uint4 *a[2];
  const uint32_t *sz[2];
  int group_size;
  long long a_stride;     // uint4 per A block
  long long sz_stride;    // u32 per A block
  int use_a_blk;
  int8_t a_blk[kMaxExperts];
  const __half *b;
  int ldb;
  const int *b_row;
  int rank;
  const uint4 *u[2];
  long long u_stride;     // uint4 per U block
  int8_t u_blk[2][kMaxExperts];
  const __half *zb[2];
  int ldz;
  const int *z_row[2];
  int epi;
  void *out[2];
  int ldo;
  long long out_split_stride;
  const float *row_scale;
  const float *col_scale;
  int ksplit;
  int m_tiles;
};

struct GemmBatch {
  GemmProblem p[2];
};

struct GemmShape {
  int am, np, bn, warps;
};

// Process-wide count of kernel launches issued by the library.
void count_launches(int n = 1);

cudaError_t launch_gemm(const GemmBatch &batch, int nprob, GemmShape shape, int n_tile_slots,
                        cudaStream_t stream);
int gemm_rows_per_cta(GemmShape shape);

// ---------------------------------------------------------------- misc
struct LrAccArgs {
  int k, r;
  const int *row_offsets;  // [M+1] (only [M] used for the count)
  int M;
  const int *rowpair_tok, *rowpair_row;
  const int32_t *topk_idx;
  const float *topk_w;
  int8_t m_of[kMaxExperts];
  const int *slot_of_pair;
  // source: per-slot fp32 z' (weights already applied) or per-colpair fp16 z times w
  const float *zslot;
  const __half *zcol;
  const int *zidx;
  __half *a;               // [rowpairs][r]
};

struct CombineArgs {
  int T, k, d, ksplit;
  long long split_stride;
  const int *slot_of_pair;
  const float *ybuf;       // [ksplit][P][d]
  const float *yshared;    // [T][d] or null
  __nv_bfloat16 *out;
};

struct ScaleGatherArgs {
  int P, d;
  const int *slot_tok;
  const float *slot_w;
  const __half *x16;
  __half *xs;              // [P][d]
};

struct SwigluArgs {
  long long n;             // P * F
  int F;
  const float *g, *u;
  const float *slot_w;
  __half *h;
};

__global__ void route_kernel(RouteArgs a);
__global__ void permute_kernel(PermuteArgs a);
__global__ void lr_accumulate_kernel(LrAccArgs a);
__global__ void combine_kernel(CombineArgs a);
__global__ void scale_gather_kernel(ScaleGatherArgs a);
__global__ void swiglu_kernel(SwigluArgs a);
__global__ void bounded_wait_kernel(int *status, int max_polls);

// ---------------------------------------------------------------- packing
__global__ void pack_codes_kernel(const uint32_t *codes, uint4 *out, int K, int d_out, int d_in);
__global__ void pack_sz_kernel(const __half *scales, const uint8_t *zeros, uint32_t *out, int K,
                               int d_out, int G);
// Fragment layout of a bf16 matrix S[R][C] (element (i, j) at src[i*rs + j*cs] of
// block b at src + b*bs) -> fp16 [B][R/16][C/16][32 lanes] uint4.
__global__ void pack_frag_kernel(const __nv_bfloat16 *src, long long bs, long long rs,
                                 long long cs, int nblk, int R, int C, uint4 *out);

}  // namespace tileq
