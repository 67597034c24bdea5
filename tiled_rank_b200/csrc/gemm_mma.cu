// Grouped mixed-input GEMM on warp-level tensor-core MMA (m16n8k16, fp16 in,
// fp32 accumulate).  This is the decode-sized path and the general fallback
// schedule for every grouped product of the TileQ forward:
//
//   residual   out[item][o] = sum_k deq(Q_e)[o][k] * B[row(item)][k]
//              with deq(Q) = s * (q - z) decoded from packed 2-bit codes straight
//              into the A fragment registers (no shared-memory round trip),
//   low-rank   + sum_i U_m[o][i] * Z[zrow(item)][i]  (K extension of the same
//              accumulators: the shared left factor of the expert's grid row),
//   F16 mode   A is a pre-packed fp16 fragment matrix (V_n^T, U blocks, shared
//              expert weights),
//
// with the epilogues: SwiGLU (gate/up pair), fp32 / fp16 store, fp32
// accumulate.  Warps tile the output features (16 rows each); every warp of
// a CTA shares one cp.async-staged tile of BN items.
#include "kernels.cuh"

namespace tileq {

namespace {

constexpr int BK = 128;
constexpr int BROW = BK + 8;  // padded smem row of B (halves): conflict-free ldmatrix

template <int AM, int NP, int BN, int WARPS, int STAGES>
struct Cfg {
  static constexpr int THREADS = WARPS * 32;
  static constexpr int NT = BN / 8;
  static constexpr int A_U4 = (AM == AM_Q2) ? 32 : 32 * 8;  // uint4 per warp per proj per stage
  static constexpr int SZ_U4 = (AM == AM_Q2) ? 16 : 0;      // uint4 of scale/zero words
  static constexpr int B_BYTES = BN * BROW * 2;
  static constexpr int A_BYTES = WARPS * NP * A_U4 * 16;
  static constexpr int SZ_BYTES = WARPS * NP * SZ_U4 * 16;
  static constexpr int STAGE_BYTES = B_BYTES + A_BYTES + SZ_BYTES;
  static constexpr int SMEM = STAGES * STAGE_BYTES;
};

template <int AM, int NP, int BN, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) gemm_mma_kernel(const __grid_constant__ GemmBatch batch) {
  using C = Cfg<AM, NP, BN, WARPS, STAGES>;
  const GemmProblem &P = batch.p[blockIdx.y];
  extern __shared__ __align__(128) uint8_t smem[];

  int bid = blockIdx.x;
  const int split = bid % P.ksplit;
  bid /= P.ksplit;
  const int mt = bid % P.m_tiles;
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
  const int o16 = mt * WARPS + warp;
  const int n16 = P.d_out >> 4;
  const bool active = o16 < n16;
  const int ablk = P.use_a_blk ? P.a_blk[grp] : grp;
  const int nkb = (P.d_in + BK - 1) / BK;  // Q2 requires d_in % BK == 0; F16 may end ragged
  const int per = (nkb + P.ksplit - 1) / P.ksplit;
  const int kb0 = min(nkb, split * per), kb1 = min(nkb, kb0 + per);

  const int g = P.group_size;
  const int G = (AM == AM_Q2) ? P.d_in / g : 1;
  const int gps = (AM == AM_Q2) ? max(1, BK / g) : 0;  // groups per stage

  auto stage_b = [&](int st) { return reinterpret_cast<__half *>(smem + st * C::STAGE_BYTES); };
  auto stage_a = [&](int st, int w, int p) {
    return reinterpret_cast<uint4 *>(smem + st * C::STAGE_BYTES + C::B_BYTES) + (w * NP + p) * C::A_U4;
  };
  auto stage_sz = [&](int st, int w, int p) {
    return reinterpret_cast<uint32_t *>(smem + st * C::STAGE_BYTES + C::B_BYTES + C::A_BYTES) +
           (w * NP + p) * C::SZ_U4 * 4;
  };

  auto load_stage = [&](int kb, int st) {
    __half *bs = stage_b(st);
    const int kvalid = min(BK, P.d_in - kb * BK);
    for (int c = threadIdx.x; c < BN * (BK / 8); c += C::THREADS) {
      const int n = c / (BK / 8), ch = c % (BK / 8);
      const bool valid = n < nitems && ch * 8 < kvalid;
      const int item = item0 + n;
      const int row = valid ? (P.b_row ? P.b_row[item] : item) : 0;
      const __half *src = valid ? P.b + (size_t)row * P.ldb + kb * BK + ch * 8 : P.b;
      cp_async16(bs + n * BROW + ch * 8, src, valid);
    }
    if (active) {
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        uint4 *as = stage_a(st, warp, p);
        if (AM == AM_Q2) {
          const uint4 *src = P.a[p] + ablk * P.a_stride + ((size_t)o16 * nkb + kb) * 32 + lane;
          cp_async16(as + lane, src, true);
          if (lane < gps * 4) {
            const int g0 = (kb * BK) / g;
            const uint32_t *ss = P.sz[p] + ablk * P.sz_stride + ((size_t)o16 * G + g0) * 16 + lane * 4;
            cp_async16(stage_sz(st, warp, p) + lane * 4, ss, true);
          }
        } else {
          const uint4 *src = P.a[p] + ablk * P.a_stride + ((size_t)o16 * (P.d_in / 16) + kb * 8) * 32 + lane;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (i * 16 < kvalid) cp_async16(as + i * 32 + lane, src + i * 32, true);
        }
      }
    }
  };

  float acc[NP][C::NT][4];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int j = 0; j < C::NT; ++j)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[p][j][v] = 0.f;

  // B fragments of one k16 step for all n8 tiles
  auto load_bfrag = [&](const __half *bs, int rowstride, int kcol, uint32_t (&bf)[C::NT][2]) {
    if constexpr (C::NT == 1) {
      uint32_t r[2];
      const int row = lane & 7, ch = (lane >> 3) & 1;
      ldmatrix_x2(r, bs + row * rowstride + kcol + ch * 8);
      bf[0][0] = r[0];
      bf[0][1] = r[1];
    } else {
#pragma unroll
      for (int j = 0; j < C::NT; j += 2) {
        uint32_t r[4];
        const int row = (j + (lane >> 4)) * 8 + (lane & 7), ch = (lane >> 3) & 1;
        ldmatrix_x4(r, bs + row * rowstride + kcol + ch * 8);
        bf[j][0] = r[0];
        bf[j][1] = r[1];
        bf[j + 1][0] = r[2];
        bf[j + 1][1] = r[3];
      }
    }
  };

  const int r0 = lane >> 2;
  // ---------------------------------------------------------------- main K loop
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (kb0 + s < kb1) load_stage(kb0 + s, s);
    cp_async_commit();
  }
  for (int it = 0; kb0 + it < kb1; ++it) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    {
      const int nxt = kb0 + it + STAGES - 1;
      if (nxt < kb1) load_stage(nxt, (it + STAGES - 1) % STAGES);
      cp_async_commit();
    }
    const int st = it % STAGES;
    const int kvalid = min(BK, P.d_in - (kb0 + it) * BK);
    if (active) {
      const __half *bs = stage_b(st);
      uint4 qa[NP];
      DqConst dq[NP];
      if (AM == AM_Q2) {
#pragma unroll
        for (int p = 0; p < NP; ++p) qa[p] = stage_a(st, warp, p)[lane];
      }
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        if (AM == AM_F16 && ks * 16 >= kvalid) break;
        uint32_t bf[C::NT][2];
        load_bfrag(bs, BROW, ks * 16, bf);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          uint32_t af[4];
          if (AM == AM_Q2) {
            if ((ks * 16) % g == 0) {
              const uint32_t *szs = stage_sz(st, warp, p) + ((ks * 16) / g) * 16;
              dq[p] = make_dq_const(szs[r0], szs[r0 + 8]);
            }
            const uint32_t words[4] = {qa[p].x, qa[p].y, qa[p].z, qa[p].w};
            const uint32_t w = words[ks >> 1] >> ((ks & 1) * 8);
            dequant_k16(w, dq[p], af);
          } else {
            const uint4 v = stage_a(st, warp, p)[ks * 32 + lane];
            af[0] = v.x; af[1] = v.y; af[2] = v.z; af[3] = v.w;
          }
#pragma unroll
          for (int j = 0; j < C::NT; ++j) mma_f16_16816(acc[p][j], af, bf[j][0], bf[j][1]);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---------------------------------------------------------------- low-rank K extension
  if (AM == AM_Q2 && P.rank > 0 && split == 0) {
    for (int rc = 0; rc < P.rank; rc += BK) {
      const int rlen = min(BK, P.rank - rc);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        __half *bs = stage_b(p);
        for (int c = threadIdx.x; c < BN * (BK / 8); c += C::THREADS) {
          const int n = c / (BK / 8), ch = c % (BK / 8);
          bool valid = n < nitems && ch * 8 < rlen;
          int zr = -1;
          if (valid) zr = P.z_row[p][item0 + n];
          valid = valid && zr >= 0;
          const __half *src = valid ? P.zb[p] + (size_t)zr * P.ldz + rc + ch * 8 : P.zb[p];
          cp_async16(bs + n * BROW + ch * 8, src, valid);
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      if (active) {
        for (int ks = 0; ks < rlen / 16; ++ks) {
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            uint32_t bf[C::NT][2];
            load_bfrag(stage_b(p), BROW, ks * 16, bf);
            const int ub = P.u_blk[p][grp];
            const uint4 v = __ldg(P.u[p] + ub * P.u_stride +
                                  ((size_t)o16 * (P.rank / 16) + (rc / 16) + ks) * 32 + lane);
            const uint32_t af[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < C::NT; ++j) mma_f16_16816(acc[p][j], af, bf[j][0], bf[j][1]);
          }
        }
      }
      __syncthreads();
    }
  }

  // ---------------------------------------------------------------- epilogue
  if (!active) return;
  const int cq = (lane & 3) * 2;
#pragma unroll
  for (int j = 0; j < C::NT; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int o = o16 * 16 + r0 + 8 * h;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int n = j * 8 + cq + cc;
        if (n >= nitems) continue;
        const int item = item0 + n;
        const int v = 2 * h + cc;
        if (P.epi == EPI_SWIGLU_H) {
          float hv = silu_f(acc[0][j][v]) * acc[NP - 1][j][v];
          if (P.row_scale) hv *= P.row_scale[item];
          reinterpret_cast<__half *>(P.out[0])[(size_t)item * P.ldo + o] = __float2half_rn(hv);
        } else if (P.epi == EPI_STORE_F32) {
          float y = acc[0][j][v];
          if (P.col_scale) y *= P.col_scale[o];
          reinterpret_cast<float *>(P.out[0])[split * P.out_split_stride + (size_t)item * P.ldo + o] = y;
        } else if (P.epi == EPI_STORE_F16) {
          float y = acc[0][j][v];
          if (P.col_scale) y *= P.col_scale[o];
          reinterpret_cast<__half *>(P.out[0])[(size_t)item * P.ldo + o] = __float2half_rn(y);
        } else if (P.epi == EPI_ACCUM_F32) {
          reinterpret_cast<float *>(P.out[0])[(size_t)item * P.ldo + o] += acc[0][j][v];
        } else {  // EPI_STORE2_F32
#pragma unroll
          for (int p = 0; p < NP; ++p)
            reinterpret_cast<float *>(P.out[p])[(size_t)item * P.ldo + o] = acc[p][j][v];
        }
      }
    }
  }
}

template <int AM, int NP, int BN>
cudaError_t launch_one(const GemmBatch &batch, int nprob, int n_tile_slots, cudaStream_t stream) {
  constexpr int WARPS = 4;
  constexpr int STAGES = (AM == AM_Q2) ? 4 : 3;
  using C = Cfg<AM, NP, BN, WARPS, STAGES>;
  auto kern = gemm_mma_kernel<AM, NP, BN, WARPS, STAGES>;
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
  const dim3 grid((unsigned)n_tile_slots * mt * ks, nprob);
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(batch);
  count_launches();
  return cudaGetLastError();
}

template <int AM, int NP>
cudaError_t launch_bn(const GemmBatch &b, int nprob, int bn, int slots, cudaStream_t s) {
  switch (bn) {
    case 8: return launch_one<AM, NP, 8>(b, nprob, slots, s);
    case 16: return launch_one<AM, NP, 16>(b, nprob, slots, s);
    case 32: return launch_one<AM, NP, 32>(b, nprob, slots, s);
    case 64: return launch_one<AM, NP, 64>(b, nprob, slots, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int gemm_rows_per_cta(GemmShape) { return 4 * 16; }

cudaError_t launch_gemm(const GemmBatch &batch, int nprob, GemmShape shape, int n_tile_slots,
                        cudaStream_t stream) {
  if (n_tile_slots <= 0 || nprob <= 0) return cudaSuccess;
  for (int i = 0; i < nprob; ++i) {
    // every problem of one launch must fit the grid computed from the maximum m_tiles/ksplit
    if (batch.p[i].m_tiles <= 0 || batch.p[i].ksplit <= 0) return cudaErrorInvalidValue;
  }
  if (shape.am == AM_Q2) {
    if (shape.np == 1) return launch_bn<AM_Q2, 1>(batch, nprob, shape.bn, n_tile_slots, stream);
    return launch_bn<AM_Q2, 2>(batch, nprob, shape.bn, n_tile_slots, stream);
  }
  if (shape.np == 1) return launch_bn<AM_F16, 1>(batch, nprob, shape.bn, n_tile_slots, stream);
  return launch_bn<AM_F16, 2>(batch, nprob, shape.bn, n_tile_slots, stream);
}

}  // namespace tileq
