// Dense fp16 GEMM on the 5th-generation tensor cores (tcgen05, TMEM), both
// operands read by TMA:
//
//   out[item][o] = epi( sum_k A[o][k] * B[item][k] )
//
// for the dense products of the TileQ forward: the projection of every token
// onto every grid column z = Sigma * (V_n^T x) (TileQ paper, section 2.2), its
// per-slot counterpart for the down projection, and the shared expert.
// A is row-major fp16 [rows][lda] (output features), B row-major fp16
// [items][ldb] (tokens or slots).  One work unit is MB row blocks of 128 (two
// projections' blocks, or consecutive blocks of one) against BN items; the MB
// MMAs of a K step share the B tile in shared memory.  Roles of one persistent
// CTA per SM:
//   warp 0      producer: 2-D TMA loads (128-byte swizzle) of A and B tiles,
//               64 K per stage, into a ring of shared-memory stages;
//   warp 1      allocates tensor memory; one elected lane issues tcgen05.mma
//               (M = 128, N = BN, K = 16, both operands in shared memory) into
//               fp32 TMEM accumulators (two buffers when they fit);
//   warps 2..9  epilogue: tcgen05.ld of the accumulators, scaling and stores,
//               two warps per TMEM lane quadrant, each half of the columns.
// Every mbarrier wait is bounded and reports TILEQ_ERR_TIMEOUT.
#include <type_traits>

#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {
namespace {

constexpr int DBK = 64;      // K per stage: one 128-byte swizzle atom
constexpr int kDenseEpw = 8;  // epilogue warps

template <int MB, int BN>
struct DenseCfg {
  static constexpr int THREADS = (2 + kDenseEpw) * 32;
  static constexpr int A_BYTES = 128 * DBK * 2;  // one row block of one stage
  static constexpr int B_BYTES = BN * DBK * 2;
  static constexpr int STAGE = MB * A_BYTES + B_BYTES;
  static constexpr int SQ_RAW = (200 * 1024) / STAGE;
  static constexpr int SQ = SQ_RAW > 8 ? 8 : SQ_RAW;
  static constexpr int ACC_COLS = MB * BN;
  static constexpr int NACC = 2 * ACC_COLS <= 512 ? 2 : 1;
  static constexpr int BAR_OFF = SQ * STAGE;
  static constexpr int SMEM = BAR_OFF + (2 * SQ + 2 * NACC + 2) * 8 + 16 + 1024;
  static_assert(SQ >= 2, "at least two stages");
  static_assert(ACC_COLS <= 512, "accumulator exceeds tensor memory");
};

// Instruction descriptor of kind::f16 with both operands K-major in shared
// memory: fp16 A and B, fp32 D, M = 128, N = n.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int MB, int BN>
__global__ void __launch_bounds__(DenseCfg<MB, BN>::THREADS, 1)
    gemm_dense_kernel(const __grid_constant__ DenseArgs P) {
  using C = DenseCfg<MB, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *q_full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *q_empty = q_full + C::SQ;
  uint64_t *acc_full = q_empty + C::SQ;  // [NACC]
  uint64_t *acc_empty = acc_full + C::NACC;
  uint64_t *drain = acc_empty + C::NACC;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto stage_a = [&](int s, int j) { return smem + s * C::STAGE + j * C::A_BYTES; };
  auto stage_b = [&](int s) { return smem + s * C::STAGE + MB * C::A_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SQ; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kDenseEpw);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::alloc(tmem_slot, 512);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  // the prologue above (barriers, TMEM) overlaps the previous kernel's tail
  pdl_wait_and_release();

  const int n_tiles = P.tiles ? *P.tile_count : (P.static_items + BN - 1) / BN;
  auto tile_of = [&](int jt) {
    return P.tiles ? P.tiles[jt] : make_int4(0, jt * BN, min(BN, P.static_items - jt * BN), 0);
  };
  const int total = n_tiles * P.m_units;
  const int nkb = P.d_in / DBK;
  // A row (tensor-map y coordinate) of row block j of unit row index ou
  auto a_row = [&](int grp, int ou, int j) {
    const int blk = P.use_a_blk ? P.a_blk[grp] : 0;
    const int rb = P.pair ? ou : ou * MB + j;
    return (blk * P.m_blocks + rb) * 128;
  };
  bool ok = true;

  if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t qi = 0;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int jt = w / P.m_units, ou = w % P.m_units;
        const int4 t = tile_of(jt);
        for (int kb = 0; kb < nkb; ++kb, ++qi) {
          const int s = qi % C::SQ;
          if (qi >= (uint32_t)C::SQ && !(ok = mbar_wait(&q_empty[s], ((qi / C::SQ) - 1) & 1, P.status))) break;
          mbar_arrive_expect_tx(&q_full[s], C::STAGE);
#pragma unroll
          for (int j = 0; j < MB; ++j) {
            int ax = kb * DBK, ay = a_row(t.x, ou, j);
            if (P.kblk) {
              // grid mode: output rows ay and K column ax fall in block (bi, bk)
              // (rows past the last block, padding of an odd row-block count, reuse the
              // last block: the epilogue drops them)
              const int bi = min(ay / P.blk_rows, P.grid_i - 1), bk = ax / P.kblk;
              ay = P.a_blk[bi * P.cell_i + bk * P.cell_k] * P.blk_rows + (ay - bi * P.blk_rows);
              ax -= bk * P.kblk;
            }
            tc::tma_load_2d(stage_a(s, j), &P.amap[P.pair ? j : 0], ax, ay, &q_full[s]);
          }
          tc::tma_load_2d(stage_b(s), &P.bmap, kb * DBK, t.y, &q_full[s]);
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (uint32_t i = qi > (uint32_t)C::SQ ? qi - C::SQ : 0; i < qi; ++i)
        mbar_wait(&q_full[i % C::SQ], (i / C::SQ) & 1, P.status);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // The whole warp waits; one elected lane issues the MMAs and commits.
    {
      // kind::f16 with both operands fp16, or both bf16 (A and B formats at bits 7 and 10)
      const uint32_t idesc = tc::idesc_f16(BN) | (P.bf16 ? ((1u << 7) | (1u << 10)) : 0u);
      uint32_t qi = 0, wi = 0;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++wi) {
        const int ab = wi % C::NACC;
        if (wi >= (uint32_t)C::NACC && !(ok = mbar_wait(&acc_empty[ab], ((wi / C::NACC) - 1) & 1, P.status))) break;
        tc::fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++qi) {
          const int s = qi % C::SQ;
          if (!(ok = mbar_wait(&q_full[s], (qi / C::SQ) & 1, P.status))) break;
          tc::fence_after();
          const uint64_t bd = tc::sdesc_sw128(smem_addr(stage_b(s)));
          const uint64_t ad0 = tc::sdesc_sw128(smem_addr(stage_a(s, 0)));
          if (tc::elect_one()) {
#pragma unroll
            for (int j = 0; j < MB; ++j) {
              // row block j sits C::A_BYTES further on; K steps of 16 inside the
              // swizzle atom advance both start addresses by 32 bytes
              const uint64_t ad = ad0 + (uint64_t)((j * C::A_BYTES) >> 4);
              const uint32_t d = tmem + ab * C::ACC_COLS + j * BN;
#pragma unroll
              for (int kk = 0; kk < DBK / 16; ++kk)
                mma_ss(d, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kb | kk) ? 1u : 0u);
            }
            tc::commit(&q_empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (tc::elect_one()) tc::commit(&acc_full[ab]);
        __syncwarp();
      }
      // all issued MMAs have retired before TMEM is released
      if (tc::elect_one()) tc::commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, P.status);
    }
  } else {
    // ============================================================ epilogue
    const int ew = warp - 2;
    const int row = (warp & 3) * 32 + lane;  // TMEM lane quadrant of this warp
    const int half = ew >> 2;                // column half of the tile
    const uint32_t lane_addr = tc::lane_base(warp);
    constexpr int COLS = BN / 2;
    constexpr int CH = COLS >= 8 ? 8 : 4;
    uint32_t wi = 0;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++wi) {
      const int jt = w / P.m_units, ou = w % P.m_units;
      const int4 t = tile_of(jt);
      const int item0 = t.y, nitems = t.z;
      const int ab = wi % C::NACC;
      if (!(ok = mbar_wait(&acc_full[ab], (wi / C::NACC) & 1, P.status))) break;
      tc::fence_after();
      int o[MB];
      float cs[MB];
#pragma unroll
      for (int j = 0; j < MB; ++j) {
        o[j] = (P.pair ? ou : ou * MB + j) * 128 + row;
        const float *c = P.col_scale[P.pair ? j : 0];
        cs[j] = c ? __ldg(c + min(o[j], P.d_out - 1)) : 1.f;
      }
      // the TMEM loads of a batch of columns go out together and are waited for
      // once (each wait lasts about as long as the queued MMAs take to drain)
      constexpr int BATCH = (MB == 1 ? 32 : 16) < COLS ? (MB == 1 ? 32 : 16) : COLS;
#pragma unroll 1
      for (int c0 = 0; c0 < COLS; c0 += BATCH) {
        float v[MB][BATCH];
#pragma unroll
        for (int cc = 0; cc < BATCH; cc += CH)
#pragma unroll
          for (int j = 0; j < MB; ++j) {
            const uint32_t addr = tmem + lane_addr + ab * C::ACC_COLS + j * BN + half * COLS + c0 + cc;
            if constexpr (CH == 8) {
              tc::ld8(addr, *reinterpret_cast<float(*)[8]>(&v[j][cc]));
            } else {
              tc::ld4(addr, *reinterpret_cast<float(*)[4]>(&v[j][cc]));
            }
          }
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int n = half * COLS + c0 + i;
          if (n >= nitems) continue;
          const size_t ib = (size_t)(item0 + n) * P.ldo;
          if (P.epi == EPI_SWIGLU_H) {
            if (o[0] < P.d_out) {
              const float rs = P.row_scale ? __ldg(P.row_scale + item0 + n) : 1.f;
              reinterpret_cast<__half *>(P.out[0])[ib + o[0]] = half_checked(silu_f(v[0][i]) * v[MB - 1][i] * rs, P.status);
            }
            continue;
          }
#pragma unroll
          for (int j = 0; j < MB; ++j) {
            if (o[j] >= P.d_out) continue;
            void *dst = P.out[P.pair ? j : 0];
            if (P.epi == EPI_STORE_F16)
              reinterpret_cast<__half *>(dst)[ib + o[j]] = half_checked(v[j][i] * cs[j], P.status);
            else if (P.epi == EPI_ACCUM_F32)
              reinterpret_cast<float *>(dst)[ib + o[j]] += v[j][i] * cs[j];
            else
              reinterpret_cast<float *>(dst)[ib + o[j]] = v[j][i] * cs[j];
          }
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }

  __syncwarp();
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

template <int MB, int BN>
cudaError_t launch_dense_one(const DenseArgs &a, int grid, cudaStream_t stream) {
  using C = DenseCfg<MB, BN>;
  auto kern = gemm_dense_kernel<MB, BN>;
  static bool configured = false;  // one attribute call per instantiation and process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM, stream, a);
  if (e != cudaSuccess) return e;
  count_launches();
  return cudaGetLastError();
}

template <int MB>
cudaError_t launch_dense_bn(const DenseArgs &a, int bn, int grid, cudaStream_t s) {
  switch (bn) {
    case 64: return launch_dense_one<MB, 64>(a, grid, s);
    case 128: return launch_dense_one<MB, 128>(a, grid, s);
    case 256: return launch_dense_one<MB, 256>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_gemm_dense(const DenseArgs &a, int mb, int bn, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  return mb == 1 ? launch_dense_bn<1>(a, bn, grid, stream) : launch_dense_bn<2>(a, bn, grid, stream);
}

}  // namespace tileq
