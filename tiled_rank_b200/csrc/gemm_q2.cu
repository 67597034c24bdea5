// Grouped 2-bit residual GEMM on warp-level tensor-core MMA (m16n8k16, fp16
// in, fp32 accumulate) for narrow tiles: the decode regime of the TileQ
// forward, where an expert sees a handful of tokens and the weight stream
// from HBM is the whole cost.
//
//   out[item][o] = epi( sum_k s*(q - z)[o][k] * B[item][k]
//                       + sum_i U_m[o][i] * B[item][ext + i] )
//
// Data movement is split by who needs the data:
//   * the 2-bit codes and the (scale, zero) words are private to one consumer
//     warp (16 output rows), so each warp streams its own slice with 16-byte
//     cp.async copies several stages ahead, with no cross-warp handshake;
//     many small independent copies keep enough bytes in flight to saturate
//     HBM, which a few 4 KB bulk copies per SM do not;
//   * the activation tile B (the tile's consecutive slots x 128 K) is shared
//     by all warps: one producer warp loads it with two 2-D TMA boxes per
//     stage (128-byte swizzle) into a ring handed over with mbarriers.
// The exact (q - z) is decoded straight into A-fragment registers (one
// AND-OR with the fp16 exponent of 1024 and one FMA per pair of weights);
// each 64/128-wide scale group accumulates into a fresh fp32 fragment that is
// folded in with its scale.  Split-K CTAs write fp32 partials; the last CTA
// of a tile sums them in split order (deterministic).
#include <type_traits>

#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

#ifdef TILEQ_TRACE
// Debug builds only: clock64 time stamps of pipeline events of CTA 0, kept
// separately for one- and two-projection launches.
__device__ unsigned long long g_q2_trace[2][6][1024];
#define Q2_TRACE(kind, idx) \
  do {                      \
    if (blockIdx.x == 0 && (idx) < 1024) g_q2_trace[NP - 1][kind][idx] = clock64(); \
  } while (0)
extern "C" int tileq_debug_q2_trace(unsigned long long *host) {
  return (int)cudaMemcpyFromSymbol(host, g_q2_trace, sizeof(g_q2_trace));
}
#else
#define Q2_TRACE(kind, idx) \
  do {                      \
  } while (0)
#endif

namespace {

constexpr int QW = 8;                    // consumer warps (16 rows each)
constexpr int QTHREADS = (QW + 1) * 32;  // + one producer warp
constexpr int QBLK = 128;                // K of one packed code block; a main stage covers two

template <int NP, int BN>
struct QCfg {
  static constexpr int NT = BN / 8;
  static constexpr int MINB = NP * NT <= 2 ? 3 : (NP * NT <= 4 ? 2 : 1);  // resident CTAs per SM
  static constexpr int BUDGET = MINB == 3 ? 74 * 1024 : (MINB == 2 ? 110 * 1024 : 200 * 1024);
  static constexpr int D = (MINB == 3 && NP == 2) ? 3 : 4;  // per-warp code/scale ring depth (stages)
  static constexpr int A_SLOT = 2 * 512;   // code bytes per warp, stage and projection (two blocks)
  static constexpr int SZ_SLOT = 2 * 128;  // (scale, zero) words: 2 blocks x 2 groups x 16 rows x 4 B
  static constexpr int BOX = BN * 128;     // one 64-wide fp16 TMA box of BN rows
  // four boxes: the 256 K of a main stage, or 128 extension columns of each of two projections
  static constexpr int B_STAGE = 4 * BOX;
  static constexpr int A_RING = QW * D * NP * A_SLOT;
  static constexpr int SZ_RING = QW * D * NP * SZ_SLOT;
  static constexpr int SB_RAW = (BUDGET - A_RING - SZ_RING - 1024) / B_STAGE;
  static constexpr int SB = SB_RAW > 8 ? 8 : SB_RAW;  // B ring stages
  static constexpr int A_OFF = SB * B_STAGE;
  static constexpr int SZ_OFF = A_OFF + A_RING;
  static constexpr int BAR_OFF = SZ_OFF + SZ_RING;
  static constexpr int SMEM = BAR_OFF + 2 * SB * 8 + 16 + 1024;  // + slack to align the base to 1024
  static_assert(SB >= 2, "shared-memory budget too small for the B ring");
  static_assert(BOX % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

__device__ __forceinline__ void q2_store(const TcArgs &a, int item, int o, float v0, float v1) {
  const size_t idx = (size_t)item * a.ldo + o;
  switch (a.epi) {
    case EPI_SWIGLU_H: {
      float h = silu_f(v0) * v1;
      if (a.row_scale) h *= a.row_scale[item];
      reinterpret_cast<__half *>(a.out[0])[idx] = __float2half_rn(h);
      break;
    }
    case EPI_STORE_F16:
      reinterpret_cast<__half *>(a.out[0])[idx] = __float2half_rn(v0);
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

template <int NP, int BN>
__global__ void __launch_bounds__(QTHREADS, QCfg<NP, BN>::MINB) gemm_q2_kernel(const __grid_constant__ TcArgs a) {
  using C = QCfg<NP, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

  int bid = blockIdx.x;
  const int split = bid % a.ksplit;
  bid /= a.ksplit;
  const int ob = bid % a.m_tiles;
  const int jt = bid / a.m_tiles;
  if (jt >= *a.tile_count) return;
  const int4 tile = a.tiles[jt];
  const int grp = tile.x, item0 = tile.y, nitems = tile.z;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n128 = a.m_tiles;
  const int nkb = a.d_in / QBLK;               // packed blocks along K
  const int nstage = (nkb + 1) / 2;            // main stages of the whole K
  const int per = (nstage + a.ksplit - 1) / a.ksplit;
  const int st0 = min(nstage, split * per), st1 = min(nstage, st0 + per);
  const int nmain = st1 - st0;
  const int next = (split == 0 && a.rank > 0) ? (a.rank + QBLK - 1) / QBLK : 0;  // 128-wide extension stages
  const int nst = nmain + next;
  const int G = a.d_in / a.group;
  const bool g64 = a.group == 64;

  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + C::SB;
  int *sflag = reinterpret_cast<int *>(empty + C::SB);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], QW);
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

  if (warp == QW) {
    // ------------------------------------------------------------ producer: B tiles by TMA
    if (lane == 0) {
      int issued = 0, s = 0;
      uint32_t par = 0;
      for (int it = 0; it < nst; ++it) {
        if (it >= C::SB && !mbar_wait(&empty[s], par ^ 1u, a.status)) break;
        uint8_t *bs = smem + s * C::B_STAGE;
        Q2_TRACE(0, it);
        if (it < nmain) {
          const int kb = 2 * (st0 + it);
          const int nbox = kb + 1 < nkb ? 4 : 2;
          mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * C::BOX));
          for (int b = 0; b < nbox; ++b) tc::tma_load_2d(bs + b * C::BOX, &a.bmap, kb * QBLK + b * 64, item0, &full[s]);
        } else {
          // low-rank extension: 128 K-extension columns of each projection
          const int e = it - nmain;
          const int nbox = (a.rank - e * QBLK) > 64 ? 2 : 1;
          mbar_arrive_expect_tx(&full[s], (uint32_t)(NP * nbox * C::BOX));
          for (int p = 0; p < NP; ++p)
            for (int b = 0; b < nbox; ++b)
              tc::tma_load_2d(bs + (p * 2 + b) * C::BOX, &a.bmap, a.ext_col[p] + e * QBLK + b * 64, item0,
                              &full[s]);
        }
        issued = it + 1;
        if (++s == C::SB) {
          s = 0;
          par ^= 1u;
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int it = max(0, issued - C::SB); it < issued; ++it)
        mbar_wait(&full[it % C::SB], (it / C::SB) & 1, a.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumer warps
    const int r0 = lane >> 2;
    const int rw = warp * 16 + r0;  // fragment rows rw and rw + 8 of the 128-row block
    const uint32_t aring = smem_addr(smem + C::A_OFF + warp * (C::D * NP * C::A_SLOT));
    const uint32_t zring = smem_addr(smem + C::SZ_OFF + warp * (C::D * NP * C::SZ_SLOT));

    // ---- copy roles.  The projections of one launch share a shape, so one
    // offset serves all of them (the launcher checks that offsets fit 32 bits).
    // codes: every lane copies its 16 bytes of each of the stage's two blocks
    uint32_t coff = (uint32_t)((((size_t)grp * n128 + ob) * nkb + 2 * st0) * 4096) + warp * 512 + lane * 16;
    // (scale, zero) words: lane -> (block h of the stage, 64-wide sub-group, 16-byte chunk)
    const int zh = g64 ? (lane >> 3) : (lane >> 2);
    const int zsub = g64 ? ((lane >> 2) & 1) : 0;
    const bool zlane = lane < (g64 ? 16 : 8);
    const uint32_t zbase = (uint32_t)(((size_t)grp * n128 + ob) * G * 128) + warp * 16 + (lane & 3) * 4;
    const uint32_t adst = aring + lane * 16;
    const uint32_t zdst = zring + zh * 128 + zsub * 64 + (lane & 3) * 16;
    // group of this lane's block 2*(st0 + ist) + zh, kept incrementally
    const int m = g64 ? 1 : a.group >> 7;  // blocks (of 128) per group
    int zgi, zrem;
    {
      const int bk = 2 * st0 + zh;
      zgi = g64 ? 2 * bk + zsub : bk / m;
      zrem = g64 ? 0 : bk % m;
    }
    int ist = 0, islot = 0;  // next main stage to copy and its ring slot
    auto issue = [&]() {
      if (ist < nmain) {
        const bool two = 2 * (st0 + ist) + 1 < nkb;  // the stage's second block exists
        const bool zcp = zlane && (zh == 0 || two);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const uint32_t ad = adst + (islot * NP + p) * C::A_SLOT;
          const uint8_t *cs = reinterpret_cast<const uint8_t *>(a.codes[p]) + coff;
          cp_async16_a(ad, cs);
          if (two) cp_async16_a(ad + 512, cs + 4096);
          if (zcp) cp_async16_a(zdst + (islot * NP + p) * C::SZ_SLOT, a.sz[p] + (zbase + (uint32_t)zgi * 128u));
        }
        coff += 2 * 4096;
        if (g64) {
          zgi += 4;
        } else {
          zrem += 2;
          while (zrem >= m) {
            zrem -= m;
            ++zgi;
          }
        }
      }
      cp_async_commit();
      ++ist;
      islot = islot == C::D - 1 ? 0 : islot + 1;
    };

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
    // one projection after the other (fewer live registers; B fragments are
    // re-read from shared memory for the second projection)
    auto block_main = [&](int slot, uint32_t bs, int h) {
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        uint32_t cw[4];
        const uint32_t sa = aring + (slot * NP + p) * C::A_SLOT + h * 512 + lane * 16;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(cw[0]), "=r"(cw[1]), "=r"(cw[2]), "=r"(cw[3])
                     : "r"(sa));
        float part[C::NT][4];
        __half2 nz[4];
        float sc0, sc8;
        auto group_consts = [&](int sub) {
          const uint32_t za = zring + (slot * NP + p) * C::SZ_SLOT + h * 128 + sub * 64 + r0 * 4;
          uint32_t u0, u8;
          asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(u0) : "r"(za));
          asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(u8) : "r"(za + 32));
          const __half2 w0 = u32_as_h2(u0), w8 = u32_as_h2(u8);
          const __half2 z0 = __high2half2(w0), z8 = __high2half2(w8);
          nz[0] = __hsub2(u32_as_h2(0xE400E400u), z0);  // -(1024 + z)
          nz[1] = __hsub2(u32_as_h2(0xDC00DC00u), z8);  // -(256 + z)
          nz[2] = __hsub2(u32_as_h2(0xD400D400u), z0);  // -(64 + z)
          nz[3] = __hsub2(u32_as_h2(0xCC00CC00u), z8);  // -(16 + z)
          sc0 = __low2float(w0);
          sc8 = __low2float(w8);
        };
        auto fold = [&]() {
#pragma unroll
          for (int j = 0; j < C::NT; ++j)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[p][j][v] = fmaf(v < 2 ? sc0 : sc8, part[j][v], acc[p][j][v]);
        };
        group_consts(0);
#pragma unroll
        for (int ks = 0; ks < QBLK / 16; ++ks) {
          const bool gstart = ks == 0 || (g64 && ks == 4);
          if (ks == 4 && g64) {
            fold();
            group_consts(1);
          }
          uint32_t bf[C::NT][2];
          load_b(bs, 2 * h, ks, bf);
          const uint32_t word = cw[ks >> 1];
          uint32_t af[4];
          dequant_qz_k16((ks & 1) ? (word >> 8) : word, nz, af);
          if (gstart) {
#pragma unroll
            for (int j = 0; j < C::NT; ++j) mma_f16_16816_z(part[j], af, bf[j][0], bf[j][1]);
          } else {
#pragma unroll
            for (int j = 0; j < C::NT; ++j) mma_f16_16816(part[j], af, bf[j][0], bf[j][1]);
          }
        }
        fold();
      }
    };

    // one extension stage: A = rows of U_m (fp16, read from global), B = 128
    // K-extension columns of each projection; FULL stages skip the bound checks
    auto stage_ext = [&](int e, uint32_t bs, int kvalid, auto full_tag) {
      constexpr bool FULL = decltype(full_tag)::value;
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
          for (int j = 0; j < C::NT; ++j) mma_f16_16816(acc[p][j], af, bf[j][0], bf[j][1]);
        }
      }
    };

    const uint32_t bring = smem_addr(smem);
#pragma unroll
    for (int i = 0; i < C::D - 1; ++i) issue();
    int cslot = 0, s = 0;
    uint32_t par = 0;
    for (int it = 0; it < nst; ++it) {
      issue();
      if (lane == 0 && (warp == 0 || warp == 7)) Q2_TRACE(warp == 0 ? 1 : 3, it);
      cp_async_wait<C::D - 1>();  // this lane's copies of stage `it` have landed
      __syncwarp();               // ... and every other lane's
      if (lane == 0 && warp == 0) Q2_TRACE(5, it);
      if (!mbar_wait(&full[s], par, a.status)) break;
      if (lane == 0 && warp == 0) Q2_TRACE(2, it);
      const uint32_t bs = bring + s * C::B_STAGE;
      if (it < nmain) {
        block_main(cslot, bs, 0);
        if (2 * (st0 + it) + 1 < nkb) block_main(cslot, bs, 1);
      } else {
        const int e = it - nmain;
        const int kvalid = min(QBLK, a.rank - e * QBLK);
        if (kvalid == QBLK)
          stage_ext(e, bs, kvalid, std::true_type{});
        else
          stage_ext(e, bs, kvalid, std::false_type{});
      }
      __syncwarp();
      if (lane == 0 && warp == 0) Q2_TRACE(4, it);
      if (lane == 0) mbar_arrive(&empty[s]);
      cslot = cslot == C::D - 1 ? 0 : cslot + 1;
      if (++s == C::SB) {
        s = 0;
        par ^= 1u;
      }
    }
    cp_async_wait<0>();

    // ---------------------------------------------------------- epilogue / partials
    const int cq = (lane & 3) * 2;
    if (a.ksplit == 1) {
#pragma unroll
      for (int j = 0; j < C::NT; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int o = ob * kRowsPerCta + warp * 16 + r0 + 8 * h;
          if (o >= a.d_out) continue;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int n = j * 8 + cq + cc;
            if (n >= nitems) continue;
            q2_store(a, item0 + n, o, acc[0][j][2 * h + cc], acc[NP - 1][j][2 * h + cc]);
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
              a.part[(((size_t)split * NP + p) * a.part_items + item0 + n) * ldp + o] = acc[p][j][2 * h + cc];
            }
          }
      __threadfence();
    }
  }

  if (a.ksplit == 1) return;
  // ------------------------------------------------------------ split-K: last CTA reduces
  __syncthreads();
  const int tile_id = jt * a.m_tiles + ob;
  if (threadIdx.x == 0) {
    const int old = atomicAdd(&a.counters[tile_id], 1);
    *sflag = (old == a.ksplit - 1);
  }
  __syncthreads();
  if (!*sflag) return;
  __threadfence();
  const int ldp = n128 * kRowsPerCta;
  for (int idx = threadIdx.x; idx < BN * kRowsPerCta; idx += QTHREADS) {
    const int n = idx / kRowsPerCta;
    const int o = ob * kRowsPerCta + idx % kRowsPerCta;
    if (n >= nitems || o >= a.d_out) continue;
    const int item = item0 + n;
    float v[2] = {0.f, 0.f};
    for (int sp = 0; sp < a.ksplit; ++sp)
#pragma unroll
      for (int p = 0; p < NP; ++p) v[p] += __ldcg(&a.part[(((size_t)sp * NP + p) * a.part_items + item) * ldp + o]);
    q2_store(a, item, o, v[0], v[NP - 1]);
  }
  if (threadIdx.x == 0) a.counters[tile_id] = 0;
}

template <int NP, int BN>
cudaError_t launch_q2(const TcArgs &a, int n_tile_slots, cudaStream_t stream) {
  using C = QCfg<NP, BN>;
  auto kern = gemm_q2_kernel<NP, BN>;
  static bool configured = false;  // one attribute call per instantiation and process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const dim3 grid((unsigned)n_tile_slots * a.m_tiles * a.ksplit);
  kern<<<grid, QTHREADS, C::SMEM, stream>>>(a);
  count_launches();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_q2(const TcArgs &a, int np, int bn, int n_tile_slots, cudaStream_t stream) {
  if (n_tile_slots <= 0) return cudaSuccess;
  if (a.m_tiles <= 0 || a.ksplit <= 0 || (a.group != 64 && a.group % 128 != 0)) return cudaErrorInvalidValue;
  // the kernel addresses codes and (scale, zero) words with 32-bit offsets
  if ((size_t)a.n_experts * a.m_tiles * 128 * (size_t)a.d_in / 4 >= ((size_t)1 << 32)) return cudaErrorInvalidValue;
  switch (bn * 4 + np) {
    case 8 * 4 + 1: return launch_q2<1, 8>(a, n_tile_slots, stream);
    case 16 * 4 + 1: return launch_q2<1, 16>(a, n_tile_slots, stream);
    case 32 * 4 + 1: return launch_q2<1, 32>(a, n_tile_slots, stream);
    case 8 * 4 + 2: return launch_q2<2, 8>(a, n_tile_slots, stream);
    case 16 * 4 + 2: return launch_q2<2, 16>(a, n_tile_slots, stream);
    case 32 * 4 + 2: return launch_q2<2, 32>(a, n_tile_slots, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tileq
