// Grouped mixed-input GEMM on the 5th-generation tensor cores (tcgen05, TMEM).
//
//   out[item][o] = sum_k deq(Q_e)[o][k] * B[item][k]  (+ sum_i U_m[o][i] * B[item][ext + i])
//
// for the residual projections of the TileQ forward (gate/up with a SwiGLU
// epilogue, down, the linear layer).  Roles of one persistent CTA per SM:
//   warp 0        producer: bulk copies of the packed 2-bit codes and group
//                 scales, 2-D TMA tiles of the activation matrix B
//                 (128-byte swizzle), into a ring of shared-memory stages;
//   warp 1        allocates tensor memory; one elected lane issues tcgen05.mma
//                 (M = 128 weight rows, N = BN items, K = 16) with A in TMEM and
//                 B in smem;
//   warps 2..     dequantisation: each thread owns one of the 128 weight rows,
//                 decodes its codes into fp16 (w = s * (q - z)) and writes them
//                 straight into the TMEM A stage with tcgen05.st; after the K
//                 loop the same warps read the fp32 accumulators (tcgen05.ld)
//                 and run the epilogue.
// The low-rank term is a K extension: after the residual K loop, the A stage
// holds rows of the shared factor U_m and B the matching columns of the item's
// z (or a) vector, accumulated into the same TMEM accumulator.
// Split-K work items write fp32 partials; the last one of a tile reduces them
// in split order.  Every mbarrier wait is bounded and reports TILEQ_ERR_TIMEOUT.
#include <type_traits>

#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int BK = 128;  // K per stage
constexpr int kDqw128 = 16;  // dequantising warps of the 128-item tiles

template <int NP, int BN, int DQW, bool Q3 = false>
struct TcCfg {
  // one-projection launches: eight more warps run the epilogue, from a second
  // accumulator buffer while the next unit's MMAs fill the first when BN <= 128
  // (two-projection accumulators fill TMEM, so there the dequantising warps
  // run the epilogue)
  static constexpr bool EW = NP == 1;
  static constexpr int NACC = EW && BN <= 128 ? 2 : 1;
  static constexpr int EPW = EW ? 8 : 0;  // two warps per TMEM lane quadrant
  static constexpr int THREADS = (2 + DQW + EPW) * 32;
  static constexpr int KPW = BK / (DQW / 4);          // K elements per dequant warp per stage
  static constexpr int CODES = NP * 128 * 32;         // packed codes of one stage (bytes)
  static constexpr int SZ = NP * 2 * 128 * 4;         // scale/zero words, up to 2 groups per stage
  static constexpr int HI = Q3 ? NP * 128 * 16 : 0;   // 3-bit codes: the high-bit plane of the stage
  static constexpr int BATOM = BN * 128;              // one 64-wide K atom of B (bytes)
  static constexpr int B = 2 * BATOM;                 // 128 K (main) or 128 extension columns of one projection
  static constexpr int QSTAGE = ((CODES + SZ + HI + B) + 1023) / 1024 * 1024;
  static_assert((CODES + SZ + HI) % 1024 == 0, "B atoms need 1024-byte alignment");
  // one-projection launches with two accumulator buffers stage the epilogue in
  // shared memory: per column half, two buffers of EBATCH items x 128 rows of
  // fp32, written out by bulk copies (one per item row) instead of one store
  // instruction per item (256-item tiles keep the shared memory for a third
  // input stage)
  static constexpr int EBATCH = 32;
  // two-projection launches (SwiGLU h in fp16, written by the dequantising
  // warps): per column quarter two buffers of 8 items x 128 rows of fp16
  static constexpr int EPI_BYTES = EW ? (BN <= 128 ? 2 * 2 * EBATCH * 128 * 4 : 0)
                                      : (BN >= 64 ? 4 * 2 * 8 * 128 * 2 : 0);
  static constexpr int SQ_RAW = (212 * 1024 - EPI_BYTES) / QSTAGE;
  static constexpr int SQ = SQ_RAW > 8 ? 8 : (SQ_RAW < 2 ? 2 : SQ_RAW);
  static constexpr int ACC_COLS = NP * BN;
  static constexpr int A_COLS = NP * (BK / 2);          // TMEM columns of one A stage
  static constexpr int SA_RAW = (512 - NACC * ACC_COLS) / A_COLS;
  static constexpr int SA = SA_RAW > 4 ? 4 : SA_RAW;
  static constexpr int EPI_OFF = SQ * QSTAGE;
  static constexpr int BAR_OFF = EPI_OFF + EPI_BYTES;
  static constexpr int SMEM_USED = BAR_OFF + (2 * SQ + 2 * SA + 8) * 8 + 64 + 1024;  // + align slack
  // at least half of the SM's shared memory: one CTA per SM, so the 512-column
  // TMEM allocation never waits for another CTA of this kernel
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static_assert(SA >= 2, "TMEM too small for two A stages");
};

// rs: the item's row scale (SwiGLU h), loaded by the caller ahead of the stores
__device__ __forceinline__ void tc_epi_store(const TcArgs &P, int item, int o, float v0, float v1, float rs) {
  const size_t idx = (size_t)item * P.ldo + o;
  if (P.epi == EPI_SWIGLU_H) {
    reinterpret_cast<__half *>(P.out[0])[idx] = half_checked(silu_f(v0) * v1 * rs, P.status);
  } else if (P.epi == EPI_STORE2_F32) {
    reinterpret_cast<float *>(P.out[0])[idx] = v0;
    reinterpret_cast<float *>(P.out[1])[idx] = v1;
  } else if (P.epi == EPI_STORE_F16) {
    reinterpret_cast<__half *>(P.out[0])[idx] = half_checked(v0, P.status);
  } else {
    reinterpret_cast<float *>(P.out[0])[idx] = v0;
  }
}

// 3-bit codes: as dq_word, with the high bit of pair (hb, i) at bits
// 2 + 2i + hb and 18 + 2i + hb of `h`, just above the 2-bit field once shifted
// by hb: the fp16 value becomes 1024 + 4^i*q (q <= 7), still exact.
__device__ __forceinline__ void dq_word3(uint32_t w, uint32_t h, const __half2 (&nz)[4], __half2 s2,
                                         uint32_t *out) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 m[4] = {u32_as_h2(0x3C003C00u), u32_as_h2(0x34003400u), u32_as_h2(0x2C002C00u),
                        u32_as_h2(0x24002400u)};
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    const uint32_t v = hb ? (w >> 8) : w;
    const uint32_t hv = hb ? (h >> 1) : h;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 x = u32_as_h2(and_or(v, 0x00030003u << (2 * i), and_or(hv, 0x00040004u << (2 * i), kMagic)));
      out[4 * hb + i] = h2_as_u32(__hmul2(__hfma2(x, m[i], nz[i]), s2));
    }
  }
}

// Decode 16 codes (one packed word) into 8 fp16x2 of s * (q - z).
__device__ __forceinline__ void dq_word(uint32_t w, const __half2 (&nz)[4], __half2 s2, uint32_t *out) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 m[4] = {u32_as_h2(0x3C003C00u), u32_as_h2(0x34003400u), u32_as_h2(0x2C002C00u),
                        u32_as_h2(0x24002400u)};
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    const uint32_t v = hb ? (w >> 8) : w;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 x = u32_as_h2(and_or(v, 0x00030003u << (2 * i), kMagic));
      out[4 * hb + i] = h2_as_u32(__hmul2(__hfma2(x, m[i], nz[i]), s2));
    }
  }
}

template <int NP, int BN, int DQW, bool Q3>
__global__ void __launch_bounds__(TcCfg<NP, BN, DQW, Q3>::THREADS, 1) gemm_tc_kernel(const __grid_constant__ TcArgs P) {
  using C = TcCfg<NP, BN, DQW, Q3>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *q_full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *q_empty = q_full + C::SQ;
  uint64_t *a_full = q_empty + C::SQ;
  uint64_t *a_empty = a_full + C::SA;
  uint64_t *acc_full = a_empty + C::SA;   // [NACC]
  uint64_t *acc_empty = acc_full + 2;     // [NACC]
  uint64_t *drain = acc_full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 6);
  int *flag = reinterpret_cast<int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto q_codes = [&](int s, int p) { return smem + s * C::QSTAGE + p * 128 * 32; };
  auto q_sz = [&](int s, int p) {
    return reinterpret_cast<uint32_t *>(smem + s * C::QSTAGE + C::CODES) + p * 2 * 128;
  };
  auto q_hi = [&](int s, int p) {
    return reinterpret_cast<const uint32_t *>(smem + s * C::QSTAGE + C::CODES + C::SZ) + p * 4 * 128;
  };
  auto q_b = [&](int s) { return smem + s * C::QSTAGE + C::CODES + C::SZ + C::HI; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SQ; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], DQW + 1);
    }
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&a_full[s], DQW);
      mbar_init(&a_empty[s], 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::EW ? C::EPW : DQW);
    }
    mbar_init(drain, 1);
    *flag = 0;
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

  const int n_tiles = *P.tile_count;
  // tile jt: (group, first item, items)
  auto tile_of = [&](int jt) { return P.tiles[jt]; };
  const int total = n_tiles * P.m_tiles * P.ksplit;
  const int nkb = P.d_in / BK;
  const int per = (nkb + P.ksplit - 1) / P.ksplit;
  const int g = P.group;
  const int G = P.d_in / g;
  const int gps = g == 64 ? 2 : 1;
  // the K extension runs one projection at a time: n_ext1 stages of 128 columns each
  const int n_ext1 = P.rank > 0 ? (P.rank + BK - 1) / BK : 0;
  const int n_ext = NP * n_ext1;
  bool ok = true;

  // the 128-row block of "projection" p of unit row index ob (row pairs: two
  // row blocks of one projection; past the last block it repeats the last one,
  // whose rows the epilogue then drops)
  auto rb_of = [&](int ob, int p) { return P.row_pair ? min(2 * ob + p, P.m_rows - 1) : ob; };
  auto decode = [&](int w, int &jt, int &ob, int &split) {
    split = w % P.ksplit;
    w /= P.ksplit;
    ob = w % P.m_tiles;
    jt = w / P.m_tiles;
  };
  auto stages_of = [&](int split, int &kb0, int &nmain, int &next) {
    kb0 = min(nkb, split * per);
    nmain = min(nkb, kb0 + per) - kb0;
    next = split == 0 ? n_ext : 0;
  };

  // ---------------------------------------------------------------- epilogue
  // Unit wi's accumulator (buffer ab) -> outputs.  COLS columns from `part *
  // COLS`, row `row` of the 128-row block; the group of `nthr` threads syncs on
  // named barrier `bar_id`; `leader` takes the split-K arrival.
  auto epilogue = [&](auto cols_c, uint32_t wi, int ab, int jt, int ob, int split, bool no_k, int item0,
                      int nitems, int row, int part, uint32_t lane_addr, int bar_id, int nthr, int tid,
                      bool leader) -> bool {
    constexpr int COLS = decltype(cols_c)::value;
    constexpr int CH = COLS >= 8 ? 8 : 4;  // columns per TMEM load
    if (!mbar_wait(&acc_full[ab], (wi / C::NACC) & 1, P.status)) return false;
    tc::fence_after();
    const int o = ob * 128 + row;
    const int ldp = P.m_tiles * 128;
    // the TMEM loads of a batch of columns go out together and are waited for
    // once: with the next unit's MMAs queued, each wait costs about as long as
    // the MMA queue takes to drain
    constexpr int BATCH = (NP == 1 ? 32 : CH) < COLS ? (NP == 1 ? 32 : CH) : COLS;
#pragma unroll 1
    for (int c0 = 0; c0 < COLS; c0 += BATCH) {
      float v[NP][BATCH];
#pragma unroll
      for (int cc = 0; cc < BATCH; cc += CH)
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const uint32_t addr = tmem + lane_addr + ab * C::ACC_COLS + p * BN + part * COLS + c0 + cc;
          if constexpr (CH == 8) {
            tc::ld8(addr, *reinterpret_cast<float(*)[8]>(&v[p][cc]));
          } else {
            tc::ld4(addr, *reinterpret_cast<float(*)[4]>(&v[p][cc]));
          }
        }
      tc::wait_ld();
      if (no_k)  // a split past the end of K contributes zeros
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
          for (int i = 0; i < BATCH; ++i) v[p][i] = 0.f;
#pragma unroll
      for (int c = 0; c < BATCH; c += CH) {
        float rs[CH];  // row scales ahead of the stores
#pragma unroll
        for (int i = 0; i < CH; ++i)
          rs[i] = P.row_scale ? __ldg(P.row_scale + item0 + min(part * COLS + c0 + c + i, nitems - 1)) : 1.f;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          const int n = part * COLS + c0 + c + i;
          if (n >= nitems) continue;
          if (P.row_pair) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
              const int op = (2 * ob + p) * 128 + row;
              if (op < P.d_out) reinterpret_cast<float *>(P.out[0])[(size_t)(item0 + n) * P.ldo + op] = v[p][c + i];
            }
          } else if (P.ksplit == 1) {
            if (o < P.d_out) tc_epi_store(P, item0 + n, o, v[0][c + i], v[NP - 1][c + i], rs[i]);
          } else {
#pragma unroll
            for (int p = 0; p < NP; ++p)
              P.part[(((size_t)split * NP + p) * P.part_items + item0 + n) * ldp + o] = v[p][c + i];
          }
        }
      }
    }
    tc::fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&acc_empty[ab]);

    if (P.ksplit > 1) {
      __threadfence();
      named_sync(bar_id, nthr);
      const int tile_id = jt * P.m_tiles + ob;
      if (leader) *flag = (atomicAdd(&P.counters[tile_id], 1) == P.ksplit - 1);
      named_sync(bar_id, nthr);
      if (*flag) {
        __threadfence();
        for (int idx = tid; idx < BN * 128; idx += nthr) {
          const int n = idx / 128, oo = ob * 128 + idx % 128;
          if (n >= nitems || oo >= P.d_out) continue;
          float r[2] = {0.f, 0.f};
          for (int sp = 0; sp < P.ksplit; ++sp)
#pragma unroll
            for (int p = 0; p < NP; ++p)
              r[p] += __ldcg(&P.part[(((size_t)sp * NP + p) * P.part_items + item0 + n) * ldp + oo]);
          tc_epi_store(P, item0 + n, oo, r[0], r[NP - 1], P.row_scale ? __ldg(P.row_scale + item0 + n) : 1.f);
        }
        if (leader) P.counters[tile_id] = 0;
      }
      named_sync(bar_id, nthr);
    }
    return true;
  };

  // ---------------------------------------------------------------- staged epilogue
  // One-projection fp32 stores (ksplit == 1): the four warps of column half
  // `part` (one per TMEM lane quadrant) move EBATCH columns at a time from TMEM
  // to a shared buffer [item][128 rows], then lane i of the half's first warp
  // writes item i's row segment with one bulk copy.  Two buffers per half: a
  // buffer is refilled once the bulk copies that read it two batches earlier
  // are done reading.
  auto epilogue_staged = [&](uint32_t wi, int ab, int ob, bool no_k, int item0, int nitems, int row, int part,
                             uint32_t lane_addr, bool leader) -> bool {
    constexpr int COLS = BN / 2, EB = C::EBATCH < COLS ? C::EBATCH : COLS;
    static_assert(EB % 8 == 0, "TMEM loads of 8 columns");
    if (!mbar_wait(&acc_full[ab], (wi / C::NACC) & 1, P.status)) return false;
    tc::fence_after();
    const bool issuer = (warp & 3) == 0;  // the half's warp of lane quadrant 0 issues the copies
    const int rows = min(128, P.d_out - ob * 128);
    float *out = reinterpret_cast<float *>(P.out[0]);
#pragma unroll 1
    for (int c0 = 0; c0 < COLS; c0 += EB) {
      const int b = (int)((wi * (COLS / EB) + c0 / EB) & 1);
      float *buf = reinterpret_cast<float *>(smem + C::EPI_OFF + (part * 2 + b) * EB * 128 * 4);
      float v[EB];
#pragma unroll
      for (int cc = 0; cc < EB; cc += 8)
        tc::ld8(tmem + lane_addr + ab * C::ACC_COLS + part * COLS + c0 + cc, *reinterpret_cast<float(*)[8]>(&v[cc]));
      tc::wait_ld();
      if (c0 + EB >= COLS) {
        // the accumulator is in registers: hand it back to the MMA warp
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
      }
      // the copies that last read this buffer (two batches ago) are done reading
      if (issuer) tc::bulk_wait_read<1>();
      named_sync(3 + part, 128);
#pragma unroll
      for (int i = 0; i < EB; ++i) buf[i * 128 + row] = no_k ? 0.f : v[i];
      tc::fence_proxy_async_smem();
      named_sync(3 + part, 128);
      if (issuer) {
        const int n = part * COLS + c0 + lane;
        if (lane < EB && n < nitems)
          tc::bulk_s2g(out + (size_t)(item0 + n) * P.ldo + ob * 128, buf + lane * 128, (uint32_t)rows * 4);
        tc::bulk_commit();
      }
    }
    return true;
  };

  // Two-projection SwiGLU epilogue (ksplit == 1) by the 16 dequantising warps:
  // the four warps of column quarter `part` move 8 columns of both
  // accumulators at a time from TMEM, store h = silu(g) * u * w in fp16 into a
  // shared buffer [item][128 rows], and lane i of the quarter's first warp
  // writes item i's row segment with one bulk copy (two buffers per quarter).
  auto epilogue_swiglu_staged = [&](uint32_t wi, int ob, bool no_k, int item0, int nitems, int row, int part,
                                    uint32_t lane_addr, bool leader) -> bool {
    if constexpr (C::EW || BN < 64) {
      return false;  // not used by these instantiations
    } else {
    constexpr int COLS = BN / 4, EB = 8;
    static_assert(COLS % EB == 0, "column quarter in batches of 8");
    if (!mbar_wait(&acc_full[0], wi & 1, P.status)) return false;
    tc::fence_after();
    const bool issuer = (warp & 3) == 2;  // dequantising warps 2, 6, 10, 14: lane quadrant 2
    const int rows = min(128, P.d_out - ob * 128);
    __half *out = reinterpret_cast<__half *>(P.out[0]);
#pragma unroll 1
    for (int c0 = 0; c0 < COLS; c0 += EB) {
      const int b = (int)((wi * (COLS / EB) + c0 / EB) & 1);
      __half *buf = reinterpret_cast<__half *>(smem + C::EPI_OFF + (part * 2 + b) * EB * 128 * 2);
      float g[EB], u[EB];
#pragma unroll
      for (int cc = 0; cc < EB; cc += 8) {
        tc::ld8(tmem + lane_addr + part * COLS + c0 + cc, *reinterpret_cast<float(*)[8]>(&g[cc]));
        tc::ld8(tmem + lane_addr + BN + part * COLS + c0 + cc, *reinterpret_cast<float(*)[8]>(&u[cc]));
      }
      tc::wait_ld();
      if (c0 + EB >= COLS) {
        // both accumulators are in registers: the next unit's MMAs may start
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[0]);
      }
      float rs[EB];
#pragma unroll
      for (int i = 0; i < EB; ++i)
        rs[i] = P.row_scale ? __ldg(P.row_scale + item0 + min(part * COLS + c0 + i, nitems - 1)) : 1.f;
      if (issuer) tc::bulk_wait_read<1>();
      named_sync(5 + part, 128);
#pragma unroll
      for (int i = 0; i < EB; ++i)
        buf[i * 128 + row] = half_checked(no_k ? 0.f : silu_f(g[i]) * u[i] * rs[i], P.status);
      tc::fence_proxy_async_smem();
      named_sync(5 + part, 128);
      if (issuer) {
        const int n = part * COLS + c0 + lane;
        if (lane < EB && n < nitems)
          tc::bulk_s2g(out + (size_t)(item0 + n) * P.ldo + ob * 128, buf + lane * 128, (uint32_t)rows * 2);
        tc::bulk_commit();
      }
    }
    return true;
    }
  };

  if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t qi = 0;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        int jt, ob, split, kb0, nmain, next;
        decode(w, jt, ob, split);
        stages_of(split, kb0, nmain, next);
        const int4 t = tile_of(jt);
        const int grp = t.x, item0 = t.y;
        for (int st = 0; st < nmain + next; ++st, ++qi) {
          const int s = qi % C::SQ;
          if (qi >= (uint32_t)C::SQ && !(ok = mbar_wait(&q_empty[s], ((qi / C::SQ) - 1) & 1, P.status))) break;
          if (st < nmain) {
            const int kb = kb0 + st;
            mbar_arrive_expect_tx(&q_full[s], NP * (128 * 32 + gps * 512) + C::HI + 2 * C::BATOM);
            for (int p = 0; p < NP; ++p) {
              const size_t cblk = (((size_t)grp * P.m_rows + rb_of(ob, p)) * nkb + kb) * (128 * 32);
              bulk_g2s(q_codes(s, p), reinterpret_cast<const uint8_t *>(P.codes[p]) + cblk, 128 * 32, &q_full[s]);
              if constexpr (Q3)
                bulk_g2s(const_cast<uint32_t *>(q_hi(s, p)),
                         reinterpret_cast<const uint8_t *>(P.codes_hi_rows[p]) + cblk / 2, 128 * 16, &q_full[s]);
              const size_t zoff = (((size_t)grp * P.m_rows + rb_of(ob, p)) * G + (kb * BK) / g) * 128;
              bulk_g2s(q_sz(s, p), P.sz[p] + zoff, gps * 512, &q_full[s]);
            }
            for (int a = 0; a < 2; ++a)
              tc::tma_load_2d(q_b(s) + a * C::BATOM, &P.bmap, kb * BK + a * 64, item0, &q_full[s]);
          } else {
            const int p = (st - nmain) / n_ext1, e = (st - nmain) % n_ext1;
            const int rlen = min(BK, P.rank - e * BK);
            const int natoms = (rlen + 63) / 64;
            mbar_arrive_expect_tx(&q_full[s], natoms * C::BATOM);
            for (int a = 0; a < natoms; ++a)
              tc::tma_load_2d(q_b(s) + a * C::BATOM, &P.bmap, P.ext_col[p] + e * BK + a * 64, item0, &q_full[s]);
          }
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (uint32_t i = qi > (uint32_t)C::SQ ? qi - C::SQ : 0; i < qi; ++i)
        mbar_wait(&q_full[i % C::SQ], (i / C::SQ) & 1, P.status);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // The whole warp runs the loop and waits on the barriers; one elected lane
    // issues the MMAs and commits, so the issuing code stays warp-uniform.
    {
      constexpr uint32_t idesc = tc::idesc_f16(BN);
      uint32_t qi = 0, ai = 0, wi = 0;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++wi) {
        int jt, ob, split, kb0, nmain, next;
        decode(w, jt, ob, split);
        stages_of(split, kb0, nmain, next);
        const int ab = wi % C::NACC;  // accumulator buffer of this unit
        if (wi >= (uint32_t)C::NACC && !(ok = mbar_wait(&acc_empty[ab], ((wi / C::NACC) - 1) & 1, P.status))) break;
        tc::fence_after();
        bool first = true;
        for (int st = 0; st < nmain + next; ++st, ++qi, ++ai) {
          const int s = qi % C::SQ, sa = ai % C::SA;
          if (!(ok = mbar_wait(&a_full[sa], (ai / C::SA) & 1, P.status))) break;
          if (!(ok = mbar_wait(&q_full[s], (qi / C::SQ) & 1, P.status))) break;
          tc::fence_after();
          const bool ext = st >= nmain;
          // an extension stage feeds one projection (pe); a main stage all of them
          const int pe = ext ? (st - nmain) / n_ext1 : 0;
          const int nk = ext ? (min(BK, P.rank - ((st - nmain) % n_ext1) * BK) + 15) / 16 : BK / 16;
          // one descriptor per stage, constant offsets (the start-address field
          // counts 16-byte units)
          const uint64_t bd0 = tc::sdesc_sw128(smem_addr(q_b(s)));
          const uint32_t a0 = tmem + C::NACC * C::ACC_COLS + sa * C::A_COLS;
          if (tc::elect_one()) {
            if (!ext) {
#pragma unroll
              for (int p = 0; p < NP; ++p) {
                const uint32_t d = tmem + ab * C::ACC_COLS + p * BN, a = a0 + p * (BK / 2);
                tc::mma_ts(d, a, bd0, idesc, first ? 0u : 1u);
#pragma unroll
                for (int kk = 1; kk < BK / 16; ++kk)
                  tc::mma_ts(d, a + kk * 8, bd0 + (uint64_t)(((kk / 4) * C::BATOM + (kk % 4) * 32) >> 4), idesc, 1u);
              }
            } else {
              const uint32_t d = tmem + ab * C::ACC_COLS + pe * BN, a = a0 + pe * (BK / 2);
              for (int kk = 0; kk < nk; ++kk)
                tc::mma_ts(d, a + kk * 8, bd0 + (uint64_t)(((kk / 4) * C::BATOM + (kk % 4) * 32) >> 4), idesc,
                           (first && kk == 0) ? 0u : 1u);
            }
            tc::commit(&a_empty[sa]);
            tc::commit(&q_empty[s]);
          }
          __syncwarp();
          first = false;
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
  } else if (warp < 2 + DQW) {
    // ============================================================ dequant (+ epilogue when NP == 2)
    const bool swiglu_staged = !C::EW && C::EPI_BYTES > 0 && DQW == 16 && P.ksplit == 1 &&
                               P.epi == EPI_SWIGLU_H && P.d_out % 8 == 0 && P.ldo % 8 == 0 &&
                               (reinterpret_cast<uintptr_t>(P.out[0]) & 15) == 0;
    const int dw = warp - 2;
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int part = dw >> 2;                  // K slice (dequant) / column slice (epilogue)
    const int row = quad * 32 + lane;          // weight row within the 128-row block
    const uint32_t lane_addr = tc::lane_base(warp);
    uint32_t qi = 0, ai = 0, wi = 0;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++wi) {
      int jt, ob, split, kb0, nmain, next;
      decode(w, jt, ob, split);
      stages_of(split, kb0, nmain, next);
      const int4 t = tile_of(jt);
      const int grp = t.x, item0 = t.y, nitems = t.z;
      // the U_m rows of this unit's extension stages, read from global memory
      // at the end of the unit: start them towards L2 now
      for (int e = 0; e < (next ? n_ext1 : 0); ++e)
#pragma unroll
        for (int p = 0; p < NP; ++p)
          if (e * BK + part * C::KPW < P.rank)
            prefetch_l2(P.u[p] + (((size_t)P.u_blk[p][grp] * P.m_rows + rb_of(ob, p)) * 128 + row) * P.rank + e * BK +
                        part * C::KPW);
      for (int st = 0; st < nmain + next; ++st, ++qi, ++ai) {
        const int s = qi % C::SQ, sa = ai % C::SA;
        if (!(ok = mbar_wait(&q_full[s], (qi / C::SQ) & 1, P.status))) break;
        const bool ext = st >= nmain;
        const int pe = ext ? (st - nmain) / n_ext1 : 0;  // the projection of an extension stage
        // decode into registers first: this overlaps the wait for a free A stage
        uint32_t vv[NP][C::KPW / 32][16];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          if (ext && p != pe) continue;
#pragma unroll
          for (int c = 0; c < C::KPW / 32; ++c) {   // chunks of 32 K elements = 16 columns
            uint32_t *v = vv[p][c];
            const int k0 = part * C::KPW + c * 32;  // K offset within the stage
            if (!ext) {
              const uint32_t *cw = reinterpret_cast<const uint32_t *>(q_codes(s, p)) + ((k0 / 32) * 128 + row) * 2;
              const int gl = g == 64 ? (k0 >> 6) : 0;
              const __half2 sz = u32_as_h2(q_sz(s, p)[gl * 128 + row]);
              const __half2 z2 = __high2half2(sz), s2 = __low2half2(sz);
              const __half2 nz[4] = {__hsub2(__float2half2_rn(-1024.f), z2), __hsub2(__float2half2_rn(-256.f), z2),
                                     __hsub2(__float2half2_rn(-64.f), z2), __hsub2(__float2half2_rn(-16.f), z2)};
              if constexpr (Q3) {
                // one high-bit word per (K slice, row): code word 1's bits rotated by 8
                const uint32_t hw = q_hi(s, p)[(k0 / 32) * 128 + row];
                dq_word3(cw[0], hw, nz, s2, v);
                dq_word3(cw[1], __funnelshift_r(hw, hw, 8), nz, s2, v + 8);
              } else {
                dq_word(cw[0], nz, s2, v);
                dq_word(cw[1], nz, s2, v + 8);
              }
            } else {
              const int e = (st - nmain) % n_ext1;
              const int kg = e * BK + k0;          // column of U
              const int ub = P.u_blk[p][grp];
              const __half *ur = P.u[p] + (((size_t)ub * P.m_rows + rb_of(ob, p)) * 128 + row) * P.rank;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint4 q4 = make_uint4(0, 0, 0, 0);
                if (kg + j * 8 < P.rank) q4 = *reinterpret_cast<const uint4 *>(ur + kg + j * 8);
                v[4 * j + 0] = q4.x;
                v[4 * j + 1] = q4.y;
                v[4 * j + 2] = q4.z;
                v[4 * j + 3] = q4.w;
              }
            }
          }
        }
        // the codes of this stage are consumed: the producer may refill it once the MMAs are done too
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_empty[s]);
        if (ai >= (uint32_t)C::SA && !(ok = mbar_wait(&a_empty[sa], ((ai / C::SA) - 1) & 1, P.status))) break;
        tc::fence_after();
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          if (ext && p != pe) continue;
          const uint32_t acol =
              tmem + lane_addr + C::NACC * C::ACC_COLS + sa * C::A_COLS + p * (BK / 2) + part * (C::KPW / 2);
#pragma unroll
          for (int c = 0; c < C::KPW / 32; ++c) tc::st16(acol + c * 16, vv[p][c]);
        }
        tc::wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[sa]);
      }
      if (!ok) break;

      if (!C::EW) {
        if (swiglu_staged) {
          if (!(ok = epilogue_swiglu_staged(wi, ob, nmain + next == 0, item0, nitems, row, part, lane_addr,
                                            dw == 0 && lane == 0)))
            break;
        } else if (!(ok = epilogue(std::integral_constant<int, BN / (DQW / 4)>{}, wi, 0, jt, ob, split,
                                   nmain + next == 0, item0, nitems, row, part, lane_addr, 1, DQW * 32,
                                   dw * 32 + lane, dw == 0 && lane == 0))) {
          break;
        }
      }
    }
    // every bulk copy of this thread has landed before the CTA exits
    if (swiglu_staged && (warp & 3) == 2) tc::bulk_wait_all();
  } else {
    // ============================================================ epilogue warps (NP == 1)
    // fp32 stores without K splits go through shared memory (rows of 16-byte multiples)
    const bool staged = C::EPI_BYTES > 0 && P.ksplit == 1 && P.epi == EPI_STORE_F32 && P.d_out % 4 == 0 && P.ldo % 4 == 0 &&
                        (reinterpret_cast<uintptr_t>(P.out[0]) & 15) == 0;
    const int ew = warp - 2 - DQW;
    const int row = (warp & 3) * 32 + lane;  // this warp's TMEM lane quadrant
    const int epart = ew >> 2;                 // column half
    const uint32_t lane_addr = tc::lane_base(warp);
    uint32_t wi = 0;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++wi) {
      int jt, ob, split, kb0, nmain, next;
      decode(w, jt, ob, split);
      stages_of(split, kb0, nmain, next);
      const int4 t = tile_of(jt);
      if (staged) {
        if (!(ok = epilogue_staged(wi, wi % C::NACC, ob, nmain + next == 0, t.y, t.z, row, epart, lane_addr,
                                   ew == 0 && lane == 0)))
          break;
      } else if (!(ok = epilogue(std::integral_constant<int, BN / (C::EW ? C::EPW / 4 : 1)>{}, wi, wi % C::NACC, jt,
                                 ob, split, nmain + next == 0, t.y, t.z, row, epart, lane_addr, 2, C::EPW * 32,
                                 ew * 32 + lane, ew == 0 && lane == 0))) {
        break;
      }
    }
    // every bulk copy of this thread has landed before the CTA exits
    if (staged && (warp & 3) == 0) tc::bulk_wait_all();
  }

  __syncwarp();
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

template <int NP, int BN, int DQW, bool Q3>
cudaError_t launch_tc_one(const TcArgs &a, int grid, cudaStream_t stream) {
  using C = TcCfg<NP, BN, DQW, Q3>;
  auto kern = gemm_tc_kernel<NP, BN, DQW, Q3>;
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

template <int NP, bool Q3>
cudaError_t launch_tc_bn(const TcArgs &a, int bn, int grid, cudaStream_t s) {
  switch (bn) {
    case 16: return launch_tc_one<NP, 16, 16, Q3>(a, grid, s);
    case 32: return launch_tc_one<NP, 32, 16, Q3>(a, grid, s);
    case 64: return launch_tc_one<NP, 64, 16, Q3>(a, grid, s);
    case 128: return launch_tc_one<NP, 128, kDqw128, Q3>(a, grid, s);
    case 256:  // one projection only: two 256-column accumulators would fill tensor memory
      if constexpr (NP == 1) return launch_tc_one<NP, 256, kDqw128, Q3>(a, grid, s);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace


int tc_smem_bytes(int np, int bn) {
  if (np == 1) {
    switch (bn) {
      case 16: return TcCfg<1, 16, 16>::SMEM;
      case 32: return TcCfg<1, 32, 16>::SMEM;
      case 64: return TcCfg<1, 64, 16>::SMEM;
      case 256: return TcCfg<1, 256, kDqw128>::SMEM;
      default: return TcCfg<1, 128, kDqw128>::SMEM;
    }
  }
  switch (bn) {
    case 16: return TcCfg<2, 16, 16>::SMEM;
    case 32: return TcCfg<2, 32, 16>::SMEM;
    case 64: return TcCfg<2, 64, 16>::SMEM;
    default: return TcCfg<2, 128, kDqw128>::SMEM;
  }
}

cudaError_t launch_gemm_tc(const TcArgs &a, int np, int bn, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  if (a.codes_hi_rows[0] != nullptr)   // 3-bit codes
    return np == 1 ? launch_tc_bn<1, true>(a, bn, grid, stream) : launch_tc_bn<2, true>(a, bn, grid, stream);
  return np == 1 ? launch_tc_bn<1, false>(a, bn, grid, stream) : launch_tc_bn<2, false>(a, bn, grid, stream);
}

}  // namespace tileq
