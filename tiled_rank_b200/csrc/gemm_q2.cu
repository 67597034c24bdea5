// Grouped 2-bit residual GEMM on warp-level tensor-core MMA (m16n8k16, fp16
// in, fp32 accumulate) for narrow tiles: the decode regime of the TileQ
// forward, where an expert sees a handful of tokens and the weight stream
// from HBM is the whole cost.
//
//   out[item][o] = epi( sum_k s*(q - z)[o][k] * B[item][k]
//                       + sum_i U_m[o][i] * B[item][ext + i] )
//
// One producer warp fills a ring of 256-wide K stages: per stage one bulk copy
// of the 2-bit codes of the CTA's 128 rows (8 KB per projection, per-lane
// fragment order), one of their (scale, zero) words, and the activation tile
// B (the tile's consecutive slots x 256 K) as four 2-D TMA boxes with 128-byte
// swizzle, all completing on one mbarrier.  Few, large copies keep enough
// bytes in flight per SM to stream HBM; eight consumer warps (16 rows each)
// only wait, decode and multiply.
// The exact (q - z) is decoded straight into A-fragment registers (one
// AND-OR with the fp16 exponent of 1024 and one FMA per pair of weights);
// each 64/128-wide scale group accumulates into a fresh fp32 fragment that is
// folded in with its scale.  Split-K CTAs write fp32 partials; the last CTA
// of a (tile, row block) sums them in split order (deterministic).
#include <type_traits>

#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int QW = 8;                    // consumer warps (16 rows each)
constexpr int QTHREADS = (QW + 1) * 32;  // + one producer warp
constexpr int QBLK = 128;                // K of one packed code block; a main stage covers two

template <int NP, int BN, bool Q3>
struct QCfg {
  static constexpr int NT = BN / 8;
  static constexpr int MINB = NP * NT <= 2 ? 3 : (NP * NT <= 4 ? 2 : 1);  // resident CTAs per SM
  static constexpr int BUDGET = MINB == 3 ? 74 * 1024 : (MINB == 2 ? 110 * 1024 : 200 * 1024);
  static constexpr int BOX = BN * 128;  // one 64-wide fp16 TMA box of BN rows
  // four boxes: the 256 K of a main stage, or 128 extension columns of each of two projections
  static constexpr int B_BYTES = 4 * BOX;
  static constexpr int A_BYTES = NP * 2 * 4096;  // codes: two 128x128 blocks per projection
  static constexpr int SZ_BYTES = NP * 2 * 1024;  // (scale, zero): per block up to two 64-wide groups
  static constexpr int H_BYTES = Q3 ? NP * 2 * 2048 : 0;  // 3-bit codes: the high-bit plane
  static constexpr int STAGE = B_BYTES + A_BYTES + SZ_BYTES + H_BYTES;
  static constexpr int S_RAW = (BUDGET - 1024 - 64) / STAGE;
  static constexpr int S = S_RAW > 8 ? 8 : S_RAW;  // ring stages
  static constexpr int BAR_OFF = S * STAGE;
  static constexpr int SMEM = BAR_OFF + 2 * S * 8 + 16 + 1024;  // + slack to align the base to 1024
  static_assert(S >= 2, "shared-memory budget too small for the ring");
  static_assert(BOX % 1024 == 0 && STAGE % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

// rs: the item's row scale (SwiGLU h), loaded by the caller ahead of the stores
__device__ __forceinline__ void q2_store(const TcArgs &a, int item, int o, float v0, float v1, float rs) {
  const size_t idx = (size_t)item * a.ldo + o;
  switch (a.epi) {
    case EPI_SWIGLU_H:
      reinterpret_cast<__half *>(a.out[0])[idx] = half_checked(silu_f(v0) * v1 * rs, a.status);
      break;
    case EPI_STORE_F16:
      reinterpret_cast<__half *>(a.out[0])[idx] = half_checked(v0, a.status);
      break;
    case EPI_STORE_F32:
      reinterpret_cast<float *>(a.out[0])[idx] = v0;
      break;
    case EPI_ACCUM_F32:
      reinterpret_cast<float *>(a.out[0])[idx] += v0;
      break;
    default:  // EPI_STORE2_F32
      reinterpret_cast<float *>(a.out[0])[idx] = v0;
      reinterpret_cast<float *>(a.out[1])[idx] = v1;
      break;
  }
}

template <int NP, int BN, bool Q3>
__global__ void __launch_bounds__(QTHREADS, QCfg<NP, BN, Q3>::MINB) gemm_q2_kernel(const __grid_constant__ TcArgs a) {
  pdl_wait_and_release();
  using C = QCfg<NP, BN, Q3>;
  constexpr int SLOT = NP * BN * kRowsPerCta;  // floats of one fp32 partial
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n128 = a.m_tiles;
  const int nkb = a.d_in / QBLK;         // packed blocks along K
  const int nstage = (nkb + 1) / 2;      // main stages (two blocks each)
  const int next = a.rank > 0 ? (a.rank + QBLK - 1) / QBLK : 0;  // 128-wide extension stages
  const int G = a.d_in / a.group;        // scale groups per row
  const bool g64 = a.group == 64;

  // one CTA per (tile, 128-row block, K split)
  int bid = blockIdx.x;
  const int split = bid % a.ksplit;
  bid /= a.ksplit;
  const int ob = bid % n128;
  const int jt = bid / n128;
  if (jt >= *a.tile_count) return;
  const int4 tile = a.tiles[jt];
  const int grp = tile.x, item0 = tile.y, nitems = tile.z;
  const int per = (nstage + a.ksplit - 1) / a.ksplit;
  const int st0 = min(nstage, split * per), st1 = min(nstage, st0 + per);
  const int nmain = st1 - st0;
  const int nst = nmain + (split == 0 ? next : 0);

  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + C::S;
  int *sflag = reinterpret_cast<int *>(empty + C::S);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], QW);
    }
    *sflag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // stage layout: [B boxes][codes: proj, block][(scale, zero): proj, block, sub-group, 128 rows]
  auto st_b = [&](int s) { return smem + s * C::STAGE; };
  auto st_a = [&](int s, int p, int h) { return smem + s * C::STAGE + C::B_BYTES + (p * 2 + h) * 4096; };
  auto st_z = [&](int s, int p, int h) {
    return smem + s * C::STAGE + C::B_BYTES + C::A_BYTES + (p * 2 + h) * 1024;
  };
  auto st_h = [&](int s, int p, int h) {
    return smem + s * C::STAGE + C::B_BYTES + C::A_BYTES + C::SZ_BYTES + (p * 2 + h) * 2048;
  };

  if (warp == QW) {
    // ------------------------------------------------------------ producer
    int issued = 0, s = 0;
    uint32_t par = 0;
    for (int it = 0; it < nst; ++it) {
      if (it >= C::S) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], par ^ 1u, a.status);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      uint8_t *bs = st_b(s);
      if (it < nmain) {
        const int kb = 2 * (st0 + it);
        const int nh = kb + 1 < nkb ? 2 : 1;  // blocks in this stage
        const uint32_t zb = g64 ? 1024 : 512;   // (scale, zero) bytes of one block
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], (uint32_t)(nh * 2 * C::BOX + NP * nh * (4096 + zb + (Q3 ? 2048 : 0))));
        __syncwarp();
        if (lane < 2 * nh) {
          tc::tma_load_2d(bs + lane * C::BOX, &a.bmap, kb * QBLK + lane * 64, item0, &full[s]);
        } else if (lane >= 8 && lane < 8 + NP) {
          const int p = lane - 8;
          const size_t blk = ((size_t)grp * n128 + ob) * nkb + kb;
          bulk_g2s(st_a(s, p, 0), reinterpret_cast<const uint8_t *>(a.codes[p]) + blk * 4096,
                   (uint32_t)(nh * 4096), &full[s]);
        } else if (lane >= 16 && lane < 16 + 2 * NP) {
          const int p = (lane - 16) >> 1, h = (lane - 16) & 1;
          if (h < nh) {
            // group of block kb + h: groups of 64 -> two consecutive, else one
            const int gi = g64 ? 2 * (kb + h) : ((kb + h) * QBLK) / a.group;
            bulk_g2s(st_z(s, p, h), a.sz[p] + (((size_t)grp * n128 + ob) * G + gi) * 128, zb, &full[s]);
          }
        } else if (Q3 && lane >= 24 && lane < 24 + NP) {
          const int p = lane - 24;
          const size_t blk = ((size_t)grp * n128 + ob) * nkb + kb;
          bulk_g2s(st_h(s, p, 0), reinterpret_cast<const uint8_t *>(a.codes_hi[p]) + blk * 2048,
                   (uint32_t)(nh * 2048), &full[s]);
        }
      } else {
        // low-rank extension: 128 K-extension columns of each projection
        const int e = it - nmain;
        const int nbox = (a.rank - e * QBLK) > 64 ? 2 : 1;
        if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(NP * nbox * C::BOX));
        __syncwarp();
        if (lane < NP * nbox) {
          const int p = lane / nbox, b = lane % nbox;
          tc::tma_load_2d(bs + (p * 2 + b) * C::BOX, &a.bmap, a.ext_col[p] + e * QBLK + b * 64, item0, &full[s]);
        }
      }
      ++issued;
      if (++s == C::S) {
        s = 0;
        par ^= 1u;
      }
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0)
      for (int i = max(0, issued - C::S); i < issued; ++i) mbar_wait(&full[i % C::S], (i / C::S) & 1, a.status);
    __syncwarp();
  } else {
  // ------------------------------------------------------------ consumer warps
  const int r0 = lane >> 2;
  const int rw = warp * 16 + r0;  // fragment rows rw and rw + 8 of the 128-row block
  const int cq = (lane & 3) * 2;

  const int ntv = (nitems + 7) / 8;  // n8 blocks holding items of this tile
  float acc[NP][C::NT][4];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int j = 0; j < C::NT; ++j)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[p][j][v] = 0.f;

  // ---- B fragments: per-lane offsets inside a swizzled box (row & 7 == lane & 7)
  // 16-byte chunk c = 2*(ks%4) + (lane/8)%2 of the box row sits at chunk c ^ (lane%8)
  uint32_t boff[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int row = (C::NT == 1 ? 0 : (lane >> 4) * 8) + (lane & 7);
    boff[q] = row * 128 + ((((q * 2) + ((lane >> 3) & 1)) ^ (lane & 7)) << 4);
  }
  // k16 step ks (0..7) of the 128-wide K slice starting at box `box0`
  auto load_b = [&](uint32_t bs, int box0, int ks, uint32_t (&bf)[C::NT][2]) {
    const uint32_t base = bs + (box0 + (ks >> 2)) * C::BOX + boff[ks & 3];
    if constexpr (C::NT == 1) {
      uint32_t r[2];
      ldmatrix_x2_a(r, base);
      bf[0][0] = r[0];
      bf[0][1] = r[1];
    } else {
#pragma unroll
      for (int j = 0; j < C::NT; j += 2) {
        uint32_t r[4];
        ldmatrix_x4_a(r, base + j * 8 * 128);
        bf[j][0] = r[0];
        bf[j][1] = r[1];
        bf[j + 1][0] = r[2];
        bf[j + 1][1] = r[3];
      }
    }
  };

  // one 128-wide block h of a main stage: 16 rows x 128 K of every projection,
  // the projections interleaved per k16 step (one B fragment load serves both,
  // and their MMA chains are independent)
  auto block_main = [&](int s, int h) {
    const uint32_t bs = smem_addr(st_b(s));
    uint32_t cw[NP][4];
    uint32_t hw[NP][2];   // 3-bit: high-bit words (each covers two of cw)
    float part[NP][C::NT][4];
    __half2 nz[NP][4];
    float sc0[NP], sc8[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint32_t sa = smem_addr(st_a(s, p, h)) + (warp * 32 + lane) * 16;
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                   : "=r"(cw[p][0]), "=r"(cw[p][1]), "=r"(cw[p][2]), "=r"(cw[p][3])
                   : "r"(sa));
      if constexpr (Q3) {
        const uint32_t sh = smem_addr(st_h(s, p, h)) + (warp * 32 + lane) * 8;
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(hw[p][0]), "=r"(hw[p][1]) : "r"(sh));
      }
    }
    auto group_consts = [&](int p, int sub) {
      const uint32_t zs = smem_addr(st_z(s, p, h)) + rw * 4;
      uint32_t u0, u8;
      asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(u0) : "r"(zs + sub * 512));
      asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(u8) : "r"(zs + sub * 512 + 32));
      const __half2 w0 = u32_as_h2(u0), w8 = u32_as_h2(u8);
      const __half2 z0 = __high2half2(w0), z8 = __high2half2(w8);
      nz[p][0] = __hsub2(u32_as_h2(0xE400E400u), z0);
      nz[p][1] = __hsub2(u32_as_h2(0xDC00DC00u), z8);
      nz[p][2] = __hsub2(u32_as_h2(0xD400D400u), z0);
      nz[p][3] = __hsub2(u32_as_h2(0xCC00CC00u), z8);
      sc0[p] = __low2float(w0);
      sc8[p] = __low2float(w8);
    };
    auto fold = [&](int p) {
#pragma unroll
      for (int j = 0; j < C::NT; ++j)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[p][j][v] = fmaf(v < 2 ? sc0[p] : sc8[p], part[p][j][v], acc[p][j][v]);
    };
#pragma unroll
    for (int p = 0; p < NP; ++p) group_consts(p, 0);
#pragma unroll
    for (int ks = 0; ks < QBLK / 16; ++ks) {
      const bool gstart = ks == 0 || (g64 && ks == 4);
      if (ks == 4 && g64) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          fold(p);
          group_consts(p, 1);
        }
      }
      uint32_t bf[C::NT][2];
      load_b(bs, 2 * h, ks, bf);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const uint32_t word = cw[p][ks >> 1];
        uint32_t af[4];
        if constexpr (Q3) {
          // high bits of word ks/2: half (ks/2)&1 of hw, rotated into place; k16 step ks&1 one bit up
          uint32_t hword = hw[p][ks >> 2];
          if ((ks >> 1) & 1) hword = __funnelshift_r(hword, hword, 8);
          if (ks & 1) hword >>= 1;
          dequant_qz3_k16((ks & 1) ? (word >> 8) : word, hword, nz[p], af);
        } else {
          dequant_qz_k16((ks & 1) ? (word >> 8) : word, nz[p], af);
        }
        if (gstart) {
#pragma unroll
          for (int j = 0; j < C::NT; ++j)
            if (j < ntv) mma_f16_16816_z(part[p][j], af, bf[j][0], bf[j][1]);
        } else {
#pragma unroll
          for (int j = 0; j < C::NT; ++j)
            if (j < ntv) mma_f16_16816(part[p][j], af, bf[j][0], bf[j][1]);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) fold(p);
  };

  // one extension stage: A = rows of U_m (fp16, read from global), B = 128
  // K-extension columns of each projection; FULL stages skip the bound checks
  auto stage_ext = [&](int e, int s, int grp, int ob, int kvalid, auto full_tag) {
    constexpr bool FULL = decltype(full_tag)::value;
    const uint32_t bs = smem_addr(st_b(s));
#pragma unroll
    for (int ks = 0; ks < QBLK / 16; ++ks) {
      if (!FULL && ks * 16 >= kvalid) break;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        uint32_t bf[C::NT][2];
        load_b(bs, 2 * p, ks, bf);
        const __half *ur = a.u[p] + (((size_t)a.u_blk[p][grp] * n128 + ob) * 128 + rw) * a.rank + e * QBLK +
                           ks * 16 + (lane & 3) * 2;
        uint32_t af[4];
        af[0] = __ldg(reinterpret_cast<const unsigned int *>(ur));
        af[1] = __ldg(reinterpret_cast<const unsigned int *>(ur + 8 * a.rank));
        af[2] = __ldg(reinterpret_cast<const unsigned int *>(ur + 8));
        af[3] = __ldg(reinterpret_cast<const unsigned int *>(ur + 8 * a.rank + 8));
#pragma unroll
        for (int j = 0; j < C::NT; ++j)
          if (j < ntv) mma_f16_16816(acc[p][j], af, bf[j][0], bf[j][1]);
      }
    }
  };

  int s = 0;
  uint32_t par = 0;
  for (int it = 0; it < nst; ++it) {
    if (!mbar_wait(&full[s], par, a.status)) break;
    if (it < nmain) {
      block_main(s, 0);
      if (2 * (st0 + it) + 1 < nkb) block_main(s, 1);
    } else {
      const int e = it - nmain;
      const int kvalid = min(QBLK, a.rank - e * QBLK);
      if (kvalid == QBLK)
        stage_ext(e, s, grp, ob, kvalid, std::true_type{});
      else
        stage_ext(e, s, grp, ob, kvalid, std::false_type{});
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == C::S) {
      s = 0;
      par ^= 1u;
    }
  }

  // ---------------------------------------------------------- epilogue / partials
  if (a.ksplit == 1) {
    float rs[C::NT][2];  // row scales first (read-only path), then the stores
#pragma unroll
    for (int j = 0; j < C::NT; ++j)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
        rs[j][cc] = a.row_scale ? __ldg(a.row_scale + item0 + min(j * 8 + cq + cc, nitems - 1)) : 1.f;
#pragma unroll
    for (int j = 0; j < C::NT; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int o = ob * kRowsPerCta + warp * 16 + r0 + 8 * h;
        if (o >= a.d_out) continue;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = j * 8 + cq + cc;
          if (n < nitems) q2_store(a, item0 + n, o, acc[0][j][2 * h + cc], acc[NP - 1][j][2 * h + cc], rs[j][cc]);
        }
      }
  } else {
    // fp32 partial of this split: [split][tile][row block][np][bn][128]
    float *mine = a.part + ((size_t)(split * (int)(gridDim.x / a.ksplit) + jt * n128 + ob)) * SLOT;
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
      for (int j = 0; j < C::NT; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
            mine[(p * BN + j * 8 + cq + cc) * kRowsPerCta + warp * 16 + r0 + 8 * h] = acc[p][j][2 * h + cc];
    __threadfence();
  }
  }  // consumer warps

  if (a.ksplit == 1) {
    return;
  }
  // ------------------------------------------------------------ split-K: last CTA reduces
  __syncthreads();
  const int unit = jt * n128 + ob;
  if (threadIdx.x == 0) *sflag = (atomicAdd(&a.counters[unit], 1) == a.ksplit - 1);
  __syncthreads();
  if (!*sflag) return;
  __threadfence();
  // four consecutive rows per thread and step (16-byte loads), all splits summed in order
  const size_t sstride = (size_t)(gridDim.x / a.ksplit) * SLOT;  // one split's partials
  const float *first = a.part + (size_t)unit * SLOT;
  for (int idx = threadIdx.x; idx < BN * (kRowsPerCta / 4); idx += QTHREADS) {
    const int n = idx / (kRowsPerCta / 4);
    const int r4 = (idx % (kRowsPerCta / 4)) * 4;
    const int o = ob * kRowsPerCta + r4;
    if (n >= nitems || o >= a.d_out) continue;
    float4 v[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    for (int sp0 = 0; sp0 < a.ksplit; sp0 += 4) {
      float4 t[4][NP];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int p = 0; p < NP; ++p)
          t[q][p] = sp0 + q < a.ksplit ? __ldcg(reinterpret_cast<const float4 *>(
                                              first + (size_t)(sp0 + q) * sstride + (p * BN + n) * kRowsPerCta + r4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          v[p].x += t[q][p].x;
          v[p].y += t[q][p].y;
          v[p].z += t[q][p].z;
          v[p].w += t[q][p].w;
        }
    }
    const float x0[4] = {v[0].x, v[0].y, v[0].z, v[0].w};
    const float x1[4] = {v[NP - 1].x, v[NP - 1].y, v[NP - 1].z, v[NP - 1].w};
    const float rsn = a.row_scale ? __ldg(a.row_scale + item0 + n) : 1.f;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      if (o + c4 < a.d_out) q2_store(a, item0 + n, o + c4, x0[c4], x1[c4], rsn);
  }
  if (threadIdx.x == 0) a.counters[unit] = 0;
}

template <int NP, int BN, bool Q3>
cudaError_t launch_q2(const TcArgs &a, int n_tile_slots, cudaStream_t stream) {
  using C = QCfg<NP, BN, Q3>;
  auto kern = gemm_q2_kernel<NP, BN, Q3>;
  static bool configured = false;  // one attribute call per instantiation and process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const cudaError_t e = launch_pdl(kern, dim3((unsigned)n_tile_slots * a.m_tiles * a.ksplit), dim3(QTHREADS), C::SMEM,
                                   stream, a);
  if (e != cudaSuccess) return e;
  count_launches();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_q2(const TcArgs &a, int np, int bn, int n_tile_slots, cudaStream_t stream) {
  if (n_tile_slots <= 0) return cudaSuccess;
  if (a.m_tiles <= 0 || a.ksplit <= 0 || (a.group != 64 && a.group % 128 != 0)) return cudaErrorInvalidValue;
  if (a.codes_hi[0] != nullptr) {   // 3-bit codes
    switch (bn * 4 + np) {
      case 8 * 4 + 1: return launch_q2<1, 8, true>(a, n_tile_slots, stream);
      case 16 * 4 + 1: return launch_q2<1, 16, true>(a, n_tile_slots, stream);
      case 32 * 4 + 1: return launch_q2<1, 32, true>(a, n_tile_slots, stream);
      case 8 * 4 + 2: return launch_q2<2, 8, true>(a, n_tile_slots, stream);
      case 16 * 4 + 2: return launch_q2<2, 16, true>(a, n_tile_slots, stream);
      case 32 * 4 + 2: return launch_q2<2, 32, true>(a, n_tile_slots, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (bn * 4 + np) {
    case 8 * 4 + 1: return launch_q2<1, 8, false>(a, n_tile_slots, stream);
    case 16 * 4 + 1: return launch_q2<1, 16, false>(a, n_tile_slots, stream);
    case 32 * 4 + 1: return launch_q2<1, 32, false>(a, n_tile_slots, stream);
    case 8 * 4 + 2: return launch_q2<2, 8, false>(a, n_tile_slots, stream);
    case 16 * 4 + 2: return launch_q2<2, 16, false>(a, n_tile_slots, stream);
    case 32 * 4 + 2: return launch_q2<2, 32, false>(a, n_tile_slots, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tileq
