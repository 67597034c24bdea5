// Streaming grouped GEMM on warp-level tensor-core MMA (m16n8k16, fp16 in, fp32
// accumulate) for the narrow fp16 products of the TileQ forward: the column
// projection z = Sigma*(V_n^T x), the down-side projection z' = Sigma*(V_n^T h),
// the shared expert and the per-expert launches of the unfused path.  A is a
// packed fp16 fragment matrix, streamed as one bulk copy per stage (32 KB per
// projection); B rows are gathered by row index into the same stage.
//
//   out[item][o] = epi( sum_k A[o][k] * B[row(item)][k] )
//
// One producer warp feeds eight consumer warps through a ring of shared-memory
// stages filled by bulk copies (cp.async.bulk) and handed over with mbarriers,
// so consumer warps never wait on each other inside the K loop.  Each consumer
// warp owns 16 output rows of the CTA's 128-row block for every projection of
// the launch (NP = 2: gate and up of the same rows, SwiGLU in registers).
// Split-K CTAs write fp32 partials; the last CTA of a tile sums them in split
// order, so the result does not depend on scheduling.
#include <type_traits>

#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int W = 8;                     // consumer warps
constexpr int THREADS = (W + 1) * 32;    // + one producer warp
constexpr int BK = 128;                  // K per stage
constexpr int BROW = BK + 8;             // padded smem row of B (halves)

template <int NP, int BN>
struct SCfg {
  static constexpr int NT = BN / 8;
  static constexpr int A_WARP = 8 * 32;  // uint4 per warp per projection and stage
  static constexpr int A_BYTES = NP * W * A_WARP * 16;
  // B stage: padded rows (row copies) or two swizzled 64-wide TMA boxes; 1024-aligned
  static constexpr int B_BYTES = (BN * BROW * 2 + 1023) / 1024 * 1024;
  static constexpr int BOX = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BUDGET = 200 * 1024;
  static constexpr int STAGES_RAW = BUDGET / STAGE;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : (STAGES_RAW < 2 ? 2 : STAGES_RAW);
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int SMEM = BAR_OFF + 2 * STAGES * 8 + 16 + 1024;  // + slack to align the base
  static constexpr int RPL = (BN + 31) / 32;  // B rows per producer lane
};

// Epilogue of one output element.  rs = the item's row scale (SwiGLU h), cs =
// the output feature's column scale; callers load both once, ahead of the
// stores (a load after a store to memory it may alias would wait for it).
__device__ __forceinline__ void epi_store(const GemmProblem &P, int item, int o, float v0, float v1, int split,
                                          float rs, float cs) {
  const size_t idx = (size_t)item * P.ldo + o;
  switch (P.epi) {
    case EPI_PARTIAL_F32:
      reinterpret_cast<float *>(P.out[0])[((size_t)split * P.part_items + item) * P.ldo + o] = v0 * cs;
      break;
    case EPI_SWIGLU_H:
      reinterpret_cast<__half *>(P.out[0])[idx] = half_checked(silu_f(v0) * v1 * rs, P.status);
      break;
    case EPI_STORE_F16:
      reinterpret_cast<__half *>(P.out[0])[idx] = half_checked(v0 * cs, P.status);
      break;
    case EPI_STORE_F32:
      reinterpret_cast<float *>(P.out[0])[idx] = v0 * cs;
      break;
    case EPI_ACCUM_F32:
      reinterpret_cast<float *>(P.out[0])[idx] += v0;
      break;
    default:  // EPI_STORE2_F32
      reinterpret_cast<float *>(P.out[0])[idx] = v0;
      reinterpret_cast<float *>(P.out[1])[idx] = v1;
      break;
  }
}

template <int NP, int BN>
__global__ void __launch_bounds__(THREADS) gemm_stream_kernel(const __grid_constant__ GemmBatch batch) {
  pdl_wait_and_release();
  using C = SCfg<NP, BN>;
  const GemmProblem &P = batch.p[blockIdx.y];
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

  int bid = blockIdx.x;
  const int split = bid % P.ksplit;
  bid /= P.ksplit;
  const int ob = bid % P.m_tiles;
  const int jt = bid / P.m_tiles;
  int grp, item0, nitems;
  if (P.tiles != nullptr) {
    int tj = jt;
    if (P.only_group >= 0) {
      tj += P.group_first_tile[P.only_group];
      if (tj >= P.group_first_tile[P.only_group + 1]) return;
    }
    if (tj >= *P.tile_count) return;
    const int4 t = P.tiles[tj];
    grp = t.x;
    item0 = t.y;
    nitems = t.z;
  } else {
    grp = 0;
    item0 = jt * BN;
    if (item0 >= P.static_items) return;
    nitems = min(BN, P.static_items - item0);
  }
  if (P.only_group >= 0 && grp != P.only_group) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ablk = P.use_a_blk ? P.a_blk[grp] : grp;
  const int nkb = (P.d_in + BK - 1) / BK;
  const int per = (nkb + P.ksplit - 1) / P.ksplit;
  const int kb0 = min(nkb, split * per), kb1 = min(nkb, kb0 + per);
  const int nst = kb1 - kb0;
  const int n128 = P.m_tiles;

  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + C::STAGES;
  int *sflag = reinterpret_cast<int *>(empty + C::STAGES);
  auto stage_a = [&](int st) { return smem + st * C::STAGE; };
  auto stage_b = [&](int st) { return reinterpret_cast<__half *>(smem + st * C::STAGE + C::A_BYTES); };

  // row copies of a ragged last K stage leave the rest of the row as it was:
  // it must read as zeros, so clear once (TMA boxes fill zeros themselves)
  if (!P.tma_b && P.d_in % BK != 0)
    for (int i = threadIdx.x; i < C::STAGES * (C::B_BYTES / 16); i += THREADS) {
      const int st = i / (C::B_BYTES / 16), j = i % (C::B_BYTES / 16);
      reinterpret_cast<uint4 *>(stage_b(st))[j] = make_uint4(0, 0, 0, 0);
    }
  // order the generic zero stores before the bulk copies (async proxy) into the same buffers
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], W);
    }
    *sflag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  float acc[NP][C::NT][4];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int j = 0; j < C::NT; ++j)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[p][j][v] = 0.f;

  if (warp == W) {
    // ------------------------------------------------------------ producer warp
    // the B rows of this tile, looked up once (lane l copies items l, l+32, ..)
    int brow[C::RPL];
#pragma unroll
    for (int j = 0; j < C::RPL; ++j) {
      const int n = lane + 32 * j;
      brow[j] = n < nitems ? (P.b_row ? P.b_row[item0 + n] : item0 + n) : 0;
    }
    int issued = 0;
    for (int it = 0; it < nst; ++it) {
      const int s = it % C::STAGES;
      if (it >= C::STAGES) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, P.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      const int kb = kb0 + it;
      const int kvalid = min(BK, P.d_in - kb * BK);
      const uint32_t bytes = (uint32_t)C::A_BYTES + (P.tma_b ? 2u * C::BOX : (uint32_t)nitems * kvalid * 2);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes);
      __syncwarp();
      if (lane < NP) {
        const int p = lane;
        const size_t blk = ((size_t)ablk * n128 + ob) * nkb + kb;
        bulk_g2s(stage_a(s) + p * W * C::A_WARP * 16, P.a[p] + blk * W * C::A_WARP, W * C::A_WARP * 16,
                 &full[s]);
      }
      if (P.tma_b) {
        if (lane >= 16 && lane < 18)
          tc::tma_load_2d(reinterpret_cast<uint8_t *>(stage_b(s)) + (lane - 16) * C::BOX, &P.bmap,
                          kb * BK + (lane - 16) * 64, item0, &full[s]);
      } else {
#pragma unroll
        for (int j = 0; j < C::RPL; ++j) {
          const int n = lane + 32 * j;
          if (n < nitems)
            bulk_g2s(stage_b(s) + n * BROW, P.b + (size_t)brow[j] * P.ldb + (size_t)kb * BK, kvalid * 2,
                     &full[s]);
        }
      }
      issued = it + 1;
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0)
      for (int it = max(0, issued - C::STAGES); it < issued; ++it)
        mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1, P.status);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumer warps
    const int r0 = lane >> 2;

    // B fragment addresses: padded rows (row copies) or swizzled 64-wide boxes
    // (TMA; 16-byte chunk c of a box row sits at chunk c ^ (row % 8), row % 8 ==
    // lane % 8).  address(j, ks) = rbase + j * rstep + tb[ks % 4] + (ks / 4) * kstep
    const int hh = (lane >> 3) & 1;
    const uint32_t rbase = P.tma_b ? (uint32_t)((C::NT == 1 ? 0 : (lane >> 4) * 8) + (lane & 7)) * 128
                                   : (uint32_t)((C::NT == 1 ? 0 : (lane >> 4) * 8) + (lane & 7)) * BROW * 2 + hh * 16;
    const uint32_t rstep = P.tma_b ? 8 * 128 : 8 * BROW * 2;
    const uint32_t kstep = P.tma_b ? (uint32_t)C::BOX : 4 * 32;
    uint32_t tb[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) tb[q] = P.tma_b ? (uint32_t)(((q * 2 + hh) ^ (lane & 7)) << 4) : (uint32_t)q * 32;

    // One stage; FULL stages run all eight k16 steps without a bound check.
    auto stage = [&](int s, int kvalid, auto full_tag) {
      constexpr bool FULL = decltype(full_tag)::value;
      const uint32_t bs = smem_addr(stage_b(s)) + rbase;
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        if (!FULL && ks * 16 >= kvalid) break;
        uint32_t bf[C::NT][2];
        const uint32_t ba = bs + tb[ks & 3] + (ks >> 2) * kstep;
        if constexpr (C::NT == 1) {
          uint32_t r[2];
          ldmatrix_x2_a(r, ba);
          bf[0][0] = r[0];
          bf[0][1] = r[1];
        } else {
#pragma unroll
          for (int j = 0; j < C::NT; j += 2) {
            uint32_t r[4];
            ldmatrix_x4_a(r, ba + (j / 2) * 2 * rstep);
            bf[j][0] = r[0];
            bf[j][1] = r[1];
            bf[j + 1][0] = r[2];
            bf[j + 1][1] = r[3];
          }
        }
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const uint4 v =
              reinterpret_cast<const uint4 *>(stage_a(s) + p * W * C::A_WARP * 16)[(warp * 8 + ks) * 32 + lane];
          const uint32_t af[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < C::NT; ++j) mma_f16_16816(acc[p][j], af, bf[j][0], bf[j][1]);
        }
      }
    };

    for (int it = 0; it < nst; ++it) {
      const int s = it % C::STAGES;
      if (!mbar_wait(&full[s], (it / C::STAGES) & 1, P.status)) break;
      const int kvalid = min(BK, P.d_in - (kb0 + it) * BK);
      if (kvalid == BK)
        stage(s, kvalid, std::true_type{});
      else
        stage(s, kvalid, std::false_type{});
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---------------------------------------------------------- epilogue / partials
    const int cq = (lane & 3) * 2;
    if (P.ksplit == 1 || P.epi == EPI_PARTIAL_F32) {
      // scales first (read-only path), then the stores
      float cs[2], rs[C::NT][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int o = min(ob * kRowsPerCta + warp * 16 + r0 + 8 * h, P.d_out - 1);
        cs[h] = P.col_scale ? __ldg(P.col_scale + o) : 1.f;
      }
#pragma unroll
      for (int j = 0; j < C::NT; ++j)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = min(j * 8 + cq + cc, nitems - 1);
          rs[j][cc] = P.row_scale ? __ldg(P.row_scale + item0 + n) : 1.f;
        }
#pragma unroll
      for (int j = 0; j < C::NT; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int o = ob * kRowsPerCta + warp * 16 + r0 + 8 * h;
          if (o >= P.d_out) continue;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int n = j * 8 + cq + cc;
            if (n >= nitems) continue;
            epi_store(P, item0 + n, o, acc[0][j][2 * h + cc], acc[NP - 1][j][2 * h + cc], split, rs[j][cc], cs[h]);
          }
        }
    } else {
      const int ldp = n128 * kRowsPerCta;
#pragma unroll
      for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int j = 0; j < C::NT; ++j)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int o = ob * kRowsPerCta + warp * 16 + r0 + 8 * h;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int n = j * 8 + cq + cc;
              if (n >= nitems) continue;
              P.part[(((size_t)split * NP + p) * P.part_items + item0 + n) * ldp + o] = acc[p][j][2 * h + cc];
            }
          }
      __threadfence();
    }
  }

  if (P.ksplit == 1 || P.epi == EPI_PARTIAL_F32) return;
  // ------------------------------------------------------------ split-K: last CTA reduces
  __syncthreads();
  const int tile_id = blockIdx.y * (int)(gridDim.x / (P.ksplit)) + jt * P.m_tiles + ob;
  if (threadIdx.x == 0) {
    const int old = atomicAdd(&P.counters[tile_id], 1);
    *sflag = (old == P.ksplit - 1);
  }
  __syncthreads();
  if (!*sflag) return;
  __threadfence();
  // four consecutive rows per thread and step (16-byte loads), all splits of
  // one step issued before they are summed in split order
  const int ldp = n128 * kRowsPerCta;
  const size_t pstride = (size_t)P.part_items * ldp;  // one (split, projection) slab
  for (int idx = threadIdx.x; idx < BN * (kRowsPerCta / 4); idx += THREADS) {
    const int n = idx / (kRowsPerCta / 4);
    const int o = ob * kRowsPerCta + (idx % (kRowsPerCta / 4)) * 4;
    if (n >= nitems || o >= P.d_out) continue;
    const int item = item0 + n;
    const float *src = P.part + (size_t)item * ldp + o;
    float4 v[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int sp0 = 0; sp0 < P.ksplit; sp0 += 8) {
      float4 t[8][NP];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int p = 0; p < NP; ++p)
          t[u][p] = sp0 + u < P.ksplit
                        ? __ldcg(reinterpret_cast<const float4 *>(src + ((size_t)(sp0 + u) * NP + p) * pstride))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          v[p].x += t[u][p].x;
          v[p].y += t[u][p].y;
          v[p].z += t[u][p].z;
          v[p].w += t[u][p].w;
        }
    }
    const float r0v[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
    const float r1v[4] = {v[NP - 1].x, v[NP - 1].y, v[NP - 1].z, v[NP - 1].w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (o + c < P.d_out)
        epi_store(P, item, o + c, r0v[c], r1v[c], 0, P.row_scale ? __ldg(P.row_scale + item) : 1.f,
                  P.col_scale ? __ldg(P.col_scale + o + c) : 1.f);
  }
  if (threadIdx.x == 0) P.counters[tile_id] = 0;
}

template <int NP, int BN>
cudaError_t launch_one(const GemmBatch &batch, int nprob, int n_tile_slots, cudaStream_t stream) {
  using C = SCfg<NP, BN>;
  auto kern = gemm_stream_kernel<NP, BN>;
  static bool configured = false;  // one attribute call per instantiation and process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int mt = 0, ks = 1;
  for (int i = 0; i < nprob; ++i) {
    mt = max(mt, batch.p[i].m_tiles);
    ks = max(ks, batch.p[i].ksplit);
  }
  for (int i = 0; i < nprob; ++i)  // the split-K tile ids assume one shape per launch
    if (batch.p[i].ksplit > 1 && (batch.p[i].m_tiles != mt || batch.p[i].ksplit != ks))
      return cudaErrorInvalidValue;
  const dim3 grid((unsigned)n_tile_slots * mt * ks, nprob);
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(THREADS), C::SMEM, stream, batch);
  if (e != cudaSuccess) return e;
  count_launches();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmBatch &batch, int nprob, GemmShape shape, int n_tile_slots,
                        cudaStream_t stream) {
  if (n_tile_slots <= 0 || nprob <= 0) return cudaSuccess;
  for (int i = 0; i < nprob; ++i)
    if (batch.p[i].m_tiles <= 0 || batch.p[i].ksplit <= 0) return cudaErrorInvalidValue;
  if (shape.np == 1) {
    switch (shape.bn) {
      case 8: return launch_one<1, 8>(batch, nprob, n_tile_slots, stream);
      case 16: return launch_one<1, 16>(batch, nprob, n_tile_slots, stream);
      case 32: return launch_one<1, 32>(batch, nprob, n_tile_slots, stream);
      case 64: return launch_one<1, 64>(batch, nprob, n_tile_slots, stream);
      case 128: return launch_one<1, 128>(batch, nprob, n_tile_slots, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (shape.bn) {
    case 8: return launch_one<2, 8>(batch, nprob, n_tile_slots, stream);
    case 16: return launch_one<2, 16>(batch, nprob, n_tile_slots, stream);
    case 32: return launch_one<2, 32>(batch, nprob, n_tile_slots, stream);
    case 64: return launch_one<2, 64>(batch, nprob, n_tile_slots, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tileq
