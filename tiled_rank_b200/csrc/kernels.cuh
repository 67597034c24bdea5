// Kernel argument structs and launch entry points shared by the .cu files.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace tileq {

// ---------------------------------------------------------------- routing
struct RouteArgs {
  const float *logits;
  const __nv_bfloat16 *x;  // may be null (route only)
  __half *x16;
  int d_x, T, K, k;
  int full_softmax;        // 1: the chosen entries of the softmax over all K logits
  int32_t *topk_idx;
  float *topk_w;
  int *zero;               // split-K arrival counters, cleared for this forward
  int nzero;
  int *status;             // device status word (TILEQ_ERR_RANGE)
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
  int *tile_counts;        // [0]: main tiles, [1]: wide tiles
  int bn_wide;             // > 0: also a table of tiles of bn_wide items
  int4 *tiles_wide;        // [P/bn_wide + K]
  int n_zproj;             // 0, 1 or 2
  int8_t n_of[2][kMaxExperts];
  int *zidx[2];            // slot -> t*N + n (row of the projected [T, N, r] tensor)
  int row_proj;            // -1 = no row designation
  int8_t m_of_row[kMaxExperts];
  int *aidx;               // slot -> 1 for the token's first slot in its grid row, else -1
  int *pcounts;            // multi-CTA sort: [CTAs][K] pairs per expert in each CTA's chunk
};

// Batches of more than kPermMultiMin pairs are sorted by kPermChunk-pair CTAs.
constexpr int kPermChunk = 1024;
constexpr int kPermChunkThreads = 256;
constexpr int kPermMultiMin = 4096;

// 16-byte chunks per thread in flight in gather_ext_kernel.
constexpr int kGatherUnroll = 4;

// ---------------------------------------------------------------- GEMM
// EPI_PARTIAL_F32: each K split stores its own fp32 partial (times col_scale) at
// out[0][(split * part_items + item) * ldo + o]; the consumer sums the splits in
// order, so no CTA waits for another and the result stays deterministic.
enum Epi { EPI_SWIGLU_H = 0, EPI_STORE_F32 = 1, EPI_STORE_F16 = 2, EPI_ACCUM_F32 = 3,
           EPI_STORE2_F32 = 4, EPI_PARTIAL_F32 = 5 };

// One grouped fp16 GEMM  out[item][o] = sum_k A_g[o][k] * B[row(item)][k],
// items grouped by tiles (group, item0, nitems).  A rows are output features
// (packed fp16 fragments [blk][R/128][K/128][8 warps][8 k16][32 lanes]); items
// are tokens / slots / (token, column) pairs.
struct GemmProblem {
  // tma_b != 0: B rows item0.. are contiguous and read through bmap (fp16,
  // box 64 x bn, 128-byte swizzle) instead of one bulk copy per row (b_row)
  alignas(64) CUtensorMap bmap;
  int tma_b;
  const int4 *tiles;
  const int *tile_count;
  int static_items;       // tiles == nullptr: one group 0 holding this many items
  int only_group;         // >= 0: tiles [group_first_tile[g], group_first_tile[g+1]) only
  const int *group_first_tile;
  int d_out, d_in;
  const uint4 *a[2];
  int use_a_blk;
  int8_t a_blk[kMaxExperts];
  const __half *b;
  int ldb;
  const int *b_row;
  int epi;
  void *out[2];
  int ldo;
  const float *row_scale;
  const float *col_scale;
  int ksplit;
  int m_tiles;
  // split-K (ksplit > 1): fp32 partials [ksplit][NP][items][m_tiles*128] and one
  // arrival counter per (item tile, row block); the last CTA of a tile reduces
  // the partials in split order and runs the epilogue.
  float *part;
  int part_items;
  int *counters;
  int *status;
};

struct GemmBatch {
  GemmProblem p[2];
};

struct GemmShape {
  int np, bn;
};

// Process-wide count of kernel launches issued by the library.
void count_launches(int n = 1);
// Record stage-boundary event `stage` of the timing hook (no-op while it is off).
void mark_stage(int stage, cudaStream_t stream);

// Launch `kern` with programmatic stream serialization: it may be scheduled
// while the previous kernel of the stream is still running and waits for it
// in the kernel (pdl_wait_and_release).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Rows of A per CTA of the streaming GEMM (eight m16 consumer warps).
constexpr int kRowsPerCta = 128;

cudaError_t launch_gemm(const GemmBatch &batch, int nprob, GemmShape shape, int n_tile_slots,
                        cudaStream_t stream);

// ---------------------------------------------------------------- tcgen05 GEMM
// Residual GEMM on the tensor cores: A = 2-bit residual of the group's expert
// (+ the grid row's U block as a K extension), B = rows of an activation matrix
// [items][ldb] read through a 2-D tensor map (box 64 x BN, 128-byte swizzle).
struct TcArgs {
  CUtensorMap bmap;
  const int4 *tiles;
  const int *tile_count;
  int m_tiles, ksplit, d_out, d_in, group, rank;
  // row_pair (two-projection kernel, ksplit 1, fp32 stores): the two
  // "projections" are row blocks 2 ob and 2 ob + 1 of one projection, which
  // share each activation tile; m_tiles counts row-block pairs and m_rows the
  // 128-row blocks of the packed layout (m_rows == m_tiles otherwise)
  int row_pair, m_rows;
  int n_experts;             // experts (blocks) in codes / sz
  int ext_col[2];            // first B column of the K extension of projection p
  const uint4 *codes[2];     // tcgen05: [K][d_out/128][d_in/128][4 slices][128 rows][8 B]
                             // warp MMA: [K][d_out/128][d_in/128][8 warps][32 lanes][16 B]
  const uint32_t *sz[2];     // [K][d_out/128][G][128 rows] {fp16 scale, fp16 zero}
  const uint2 *codes_hi[2];  // 3-bit high plane, warp MMA: [K][d_out/128][d_in/128][8 warps][32 lanes][8 B];
                             // null for 2-bit codes
  const uint32_t *codes_hi_rows[2];  // 3-bit high plane, tcgen05: [K][d_out/128][d_in/128][4 slices][128 rows]
                                     // u32; null for 2-bit codes
  const __half *u[2];        // [M][pad128(d_out)][rank] fp16
  int8_t u_blk[2][kMaxExperts];
  int epi;
  void *out[2];
  int ldo;
  const float *row_scale;
  float *part;
  int part_items;
  int *counters;
  int *status;
};

cudaError_t launch_gemm_tc(const TcArgs &a, int np, int bn, int grid, cudaStream_t stream);

// Residual GEMM of the decode regime on tcgen05 (gemm_dq.cu): narrow item
// tiles (16, 32 or 64 items), the exact q - z of each 2-bit code in fp16 as
// the A operand in tensor memory, one fp32 accumulator per 128-wide K block
// (scale group) folded into registers with its scale, and stream-K work
// division: the (tile, row block, round) space is cut into gridDim.x equal
// ranges; a (tile, row block) unit split between CTAs is summed, in CTA
// order, by the CTA that finishes it last.  Groups are multiples of 128.
// A round covers two slices: gate and up of one 128-wide K block (np = 2) or
// two consecutive K blocks of one projection (np = 1); the low-rank K
// extension follows the residual rounds of each unit.
struct DqArgs {
  alignas(64) CUtensorMap bmap;  // B: fp16 activation rows [items][ldb], box 64 x bn, 128-byte swizzle;
                                 // fp8 mode: the e4m3 pieces [items][2][d_in] bytes, box 128 x bn
  alignas(64) CUtensorMap bmap_ext;  // fp8 mode: the fp16 rows holding the extension columns
  int f8;                        // fp8 mode (np = 2): A = e4m3 (q - z), B = two e4m3 pieces of x * 2^e
  const float *xs;               // fp8 mode: per item 2^-e
  const int4 *tiles;             // (expert, first item, items)
  const int *tile_count;
  int max_tiles;                 // capacity of tiles (bounds the rounds of a CTA)
  int m_tiles, d_out, d_in, group, rank;
  int ext_col[2];                // first B column of projection p's K extension
  const uint32_t *codes[2];      // tcgen05 row layout of the codes (qw)
  const uint32_t *sz[2];         // [K][d_out/128][G][128 rows] {fp16 scale, fp16 zero}
  const __half *u[2];            // [M][pad128(d_out)][rank] fp16
  int8_t u_blk[2][kMaxExperts];
  int epi;                       // np = 2: EPI_SWIGLU_H (fp16 h) or EPI_STORE2_F32 (gate, up in fp32);
                                 // np = 1: EPI_STORE_F32
  void *out;
  void *out2;                    // EPI_STORE2_F32: the up projection
  int ldo;
  const float *row_scale;        // per item (SwiGLU h)
  float *part;                   // split units: [gridDim.x][2][np][bn][128] fp32
  int *counters;                 // one zeroed arrival count per (tile, row block)
  int *status;
  // np = 1 with combine: out is the fp32 per-slot buffer [items][ldo]; the
  // last of a token's top_k slots to finish a row block writes
  // out_tok[t][o] = bf16(sum over the token's slots in slot order (+ yshared[t][o]))
  int combine;
  int top_k;
  const int *slot_tok;           // [items] token of each slot
  const int *slot_of_pair;       // [T * top_k]
  const float *yshared;          // [T][ldo] or null
  __nv_bfloat16 *out_tok;        // [T][ldo]
  int *tok_counters;             // [T][m_tiles], zeroed
};
cudaError_t launch_gemm_dq(const DqArgs &a, int np, int bn, cudaStream_t stream);
int dq_grid();
// Whether every CTA's rounds of a launch over at most max_tiles tiles fit the
// kernel's per-CTA round table.
bool dq_fits(int max_tiles, int m_tiles, int d_in, int rank);

// Dense fp16 GEMM on tcgen05 with both operands read by TMA (gemm_dense.cu).
// A: fp16 row-major, tensor maps amap[j] (box 64 x 128, 128-byte swizzle);
// B: fp16 item rows, bmap (box 64 x bn).  A work unit is MB row blocks of 128
// against one item tile: pair != 0: block `ou` of amap[0] and of amap[1]
// (two projections sharing B; epilogue EPI_STORE2_F32 or EPI_SWIGLU_H),
// else blocks MB*ou .. MB*ou+MB-1 of amap[0].  The A row of block rb of a tile
// of group g is (a_blk[g] * m_blocks + rb) * 128 when use_a_blk, else rb * 128.
struct DenseArgs {
  alignas(64) CUtensorMap amap[2];
  alignas(64) CUtensorMap bmap;
  const int4 *tiles;      // (group, first item, items) or nullptr: static_items in tiles of bn
  const int *tile_count;
  int static_items;
  int pair;
  int m_units;            // units per item tile
  int m_blocks;           // row blocks of one A block (cdiv(d_out, 128))
  int use_a_blk;
  int8_t a_blk[kMaxExperts];
  // grid mode (kblk > 0): A is a grid of blocks of blk_rows output rows x kblk
  // K columns, block (i, k) stored as the matrix a_blk[i * cell_i + k * cell_k]
  // of the array [blocks][blk_rows][kblk] (blk_rows a multiple of 128, kblk of 64)
  int kblk, blk_rows, cell_i, cell_k, grid_i;  // grid_i: blocks along the output rows
  int bf16;               // operands bf16 instead of fp16
  int d_out, d_in;        // d_in a multiple of 64
  int epi;
  void *out[2];
  int ldo;
  const float *col_scale[2];
  const float *row_scale;
  int *status;
};

cudaError_t launch_gemm_dense(const DenseArgs &a, int mb, int bn, int grid, cudaStream_t stream);
// 2-D tensor map over 2-byte elements [rows][ld] (cols used), box 64 x box_rows,
// 128-byte swizzle (api.cu), and the item-tile width the dense products use.
bool tensor_map_2b(CUtensorMap *m, const void *base, int rows, int cols, int ld, int box_rows);
int dense_tile_items(int items, int m_units);

// The same residual GEMM for narrow tiles (bn 8, 16 or 32) on warp-level MMA:
// codes[p] in the per-lane fragment layout of pack_codes_kernel, B through
// bmap (box 64 x bn).  One CTA per (tile slot, 128-row block, K split); with
// ksplit > 1, part holds one [np][bn][128] fp32 partial per CTA and counters
// one zeroed arrival count per (tile slot, row block).
cudaError_t launch_gemm_q2(const TcArgs &a, int np, int bn, int n_tile_slots, cudaStream_t stream);
int tc_smem_bytes(int np, int bn);

// ---------------------------------------------------------------- misc
struct GatherExtArgs {
  int P, d, r, ld;            // x_ext[s] = [x16[tok(s)] (d) | z0[zidx0[s]] (r) | z1[zidx1[s]] (r)]
  int T, k;                   // x part token-major: row t read once, written to its k slots
  const int *slot_of_pair;    // [T*k]
  int zld;                    // row stride of z0 / z1 (elements)
  int zks;                    // z0 / z1 are fp32 partials [zks][rows][zld], summed in order
  long long zsplit;           // elements between two partials
  const int *slot_tok;
  const __half *x16;
  const float *z[2];
  const int *zidx[2];
  __half *out;
  int *status;
};

// The activations of the fp8 decode GEMM (gate/up), one CTA per token t:
// with e_t the power of two that puts max|x_t| in [128, 256), each slot of the
// token gets x * 2^e_t as two e4m3 pieces (x8[slot][0][k] + x8[slot][1][k]:
// the rounded value and its rounded remainder; exact for every element within
// 2^-9 of the row maximum), the elements of each 16-wide block stored in the
// order k = 4*(s%4) + s/4 of the decoded weights (the block's 4 x 4 transpose),
// xs[slot] = 2^-e_t, and its z rows (sum of the K-split partials) times 2^e_t
// in fp16 into the extension columns d .. d + nz*r of xext.
struct GatherX8Args {
  int T, k, d, r, ld;
  const int *slot_of_pair;   // [T*k]
  const __half *x16;         // [T][d]
  uint8_t *x8;               // [P][2][d]
  float *xs;                 // [P]
  const float *z[2];         // fp32 partials [zks][rows][zld], or null
  const int *zidx[2];        // slot -> row of the projected [T, N, r] tensor
  int zld, zks;
  long long zsplit;
  __half *xext;              // [P][ld]
  int *status;
};

// Row accumulation, written per slot into the K-extension columns of the
// activation matrix: the designated slot of each (token, grid row) gets a_{t,m},
// every other slot zeros.
struct LrAccArgs {
  int P, k, r;
  const int32_t *sorted_pairs;
  const int *aidx;         // slot -> >= 0 for the token's first slot in its grid row, else -1
  const int32_t *topk_idx;
  const float *topk_w;
  int8_t m_of[kMaxExperts];
  const int *slot_of_pair;
  // source: fp32 rows of the projected [T, N, r] tensor (stride zld) times w
  // (the linear layer), or per-slot fp32 rows with the weight already applied
  // (zslot; unused by the forward); both as zks partials (zsplit elements
  // apart) summed in order
  const float *zslot;
  const float *zcol;
  const int *zidx;
  int zld;
  int zks;
  long long zsplit;
  __half *out;             // [P][ld], columns col .. col+r-1
  int ld, col;
  int *status;
};

struct CombineArgs {
  int T, k, d;
  const int *slot_of_pair;
  const float *ybuf;       // [P][d]
  const float *yshared;    // [T][d] or null
  __nv_bfloat16 *out;
};

struct ScaleGatherArgs {
  int P, d, ld;
  const int *slot_tok;
  const float *slot_w;
  const __half *x16;
  __half *xs;              // [P][ld], columns 0 .. d-1
};

struct SwigluArgs {
  long long n;             // P * F
  int F, ldh;
  const float *g, *u;
  const float *slot_w;
  __half *h;               // [P][ldh]
  int *status;
};

__global__ void route_kernel(RouteArgs a);
__global__ void route_permute_kernel(RouteArgs ra, PermuteArgs a);
__global__ void permute_count_kernel(PermuteArgs a);
__global__ void permute_scatter_kernel(PermuteArgs a);
__global__ void lr_accumulate_kernel(LrAccArgs a);
static_assert(kMaxTopK == 8, "launch_combine instantiates top-k 1..8");
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t stream);
__global__ void scale_gather_kernel(ScaleGatherArgs a);
__global__ void gather_ext_kernel(GatherExtArgs a);
__global__ void gather_x8_kernel(GatherX8Args a);
__global__ void swiglu_kernel(SwigluArgs a);
__global__ void bounded_wait_kernel(int *status, int max_polls);

// ---------------------------------------------------------------- packing
// Packed layouts (rows padded to a multiple of 128, K to a multiple of 16*kb):
//   codes  [blk][R/128][d_in/128][8 warps][32 lanes] uint4
//   sz     [blk][R/128][G][8 warps][16 rows] uint32 {fp16 scale, fp16 zero}
//   frag   [blk][R/128][C/(16*kb)][8 warps][kb k16 steps][32 lanes] uint4 (fp16 A fragments)
__global__ void pack_codes_kernel(const uint32_t *codes, uint4 *out, int K, int d_out, int d_in);
__global__ void pack_codes_hi_kernel(const uint32_t *hi, uint2 *out, int K, int d_out, int d_in);
__global__ void pack_codes_tc_hi_kernel(const uint32_t *hi, uint32_t *out, int K, int d_out, int d_in);
__global__ void pack_sz_kernel(const __half *scales, const uint8_t *zeros, uint32_t *out, int K,
                               int d_out, int G, int bits);
// Element (i, j) of block b of a bf16 matrix S[R][C] is src[b*bs + i*rs + j*cs].
__global__ void pack_frag_kernel(const __nv_bfloat16 *src, long long bs, long long rs,
                                 long long cs, int nblk, int R, int C, int kb, uint4 *out);
// 2-bit codes -> [K][R/128][d_in/128][4 K slices][128 rows][2 words]: word wi of
// slice part of a row holds elements 32*part + 16*wi .. +15 of the 128-wide block,
// pair p = (2p, 2p+1) at bits (2(p%4) + 8(p/4), 16 + 2(p%4) + 8(p/4)).  One warp
// reading one slice of 32 consecutive rows touches 256 contiguous bytes.
__global__ void pack_codes_tc_kernel(const uint32_t *codes, uint32_t *out, int K, int d_out, int d_in);
// bf16 [nblk][R][C] -> fp16 [nblk][pad128(R)][C] (zero rows appended).
__global__ void pack_vt_rows_kernel(const __nv_bfloat16 *V, int N, int r, int d_in, __half *out);
__global__ void expand_sigma_kernel(const float *sigma, int r, int rp, int n, float *out);
__global__ void pack_rows_f16_kernel(const __nv_bfloat16 *src, int nblk, int R, int C, __half *out);

__host__ __device__ inline int pad128(int x) { return (x + 127) / 128 * 128; }

}  // namespace tileq
