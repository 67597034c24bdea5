// Residual GEMM of the decode regime (a handful of tokens per expert) on the
// 5th-generation tensor cores, for the TileQ forward:
//
//   out[item][o] = epi( sum_k s*(q - z)[o][k] * B[item][k]  +  sum_i U_m[o][i] * B[item][ext + i] )
//
// At decode the weight stream from HBM is the whole cost, so the kernel is
// built around bytes in flight and instructions per weight:
//   * the A operand is the exact q - z of each 2-bit code in fp16 (one AND-OR
//     with the fp16 exponent of 1024 and one FMA per pair of weights), written
//     to tensor memory; the tensor cores do every multiply (TS-form
//     tcgen05.mma, M = 128 weight rows, N = 16..64 items);
//   * every 128-wide K block (one scale group, or part of one) accumulates
//     into its own fp32 accumulator in tensor memory; the decoding warps fold
//     it into registers with the group scale two rounds later (w = s*(q - z)
//     is never rounded);
//   * a round = two slices of 128 K: gate and up of one K block (np = 2) or
//     two consecutive K blocks of one projection (np = 1); the MMA warp waits
//     on one barrier and commits once per round;
//   * stream-K: the (tile, row block, round) space is cut into gridDim.x equal
//     contiguous ranges, one per CTA (one CTA per SM).  A (tile, row block)
//     unit cut between CTAs leaves fp32 pieces that the CTA finishing last
//     sums in CTA order (deterministic), so every SM streams the same number
//     of weight bytes whatever the routing.
// The low-rank term is a K extension: after a unit's residual rounds, the A
// slot holds rows of the grid row's U_m (fp16, read from global memory) and B
// the matching z (or a) columns of the item rows, with scale 1.
//
// Warp roles (18 warps): warp 0 producer (bulk copies of the codes and their
// (scale, zero) words, 2-D TMA boxes of B into a ring of stages), warp 1 MMA
// issuer (the whole warp waits, one elected lane issues and commits), warps
// 2..17 decode and epilogue: warp w works on TMEM lane quadrant w % 4 (32
// weight rows), slice ((w - 2) / 4) / 2 and K half / column half (w - 2) / 4 % 2.
// Every wait is bounded and reports TILEQ_ERR_TIMEOUT.
#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int DQ_DW = 16;                     // decode / epilogue warps
constexpr int DQ_THREADS = (2 + DQ_DW) * 32;  // + producer + MMA issuer
constexpr int DQ_GRID = 148;                  // one CTA per SM

template <int NP, int BN>
struct DqCfg {
  static constexpr int ATOM = BN * 128;                // one 64-wide fp16 K atom of B: BN rows x 128 B
  static constexpr int B_BYTES = 4 * ATOM;             // up to four atoms per round
  static constexpr int CODES = 2 * 4096;               // two 128 x 128 blocks of 2-bit codes
  static constexpr int SZ = 2 * 512;                   // their (scale, zero) words
  static constexpr int STAGE = (B_BYTES + CODES + SZ + 1023) / 1024 * 1024;
  static constexpr int XBUF = 128 * BN * 4;            // unit-end exchange between the two slices
  static constexpr int NS_RAW = (200 * 1024 - XBUF) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;   // ring stages
  static constexpr int XBUF_OFF = NS * STAGE;
  static constexpr int BAR_OFF = XBUF_OFF + XBUF;
  static constexpr int SMEM = BAR_OFF + (2 * NS + 5) * 8 + 16 + BN * 4 + 1024;  // + slack to align the base
  static constexpr int ACC_COLS = 2 * BN;             // one accumulator slot: two slices
  static constexpr int ACC0 = 256;                     // TMEM: A slots at 0 and 128, accumulators from 256
  static_assert(NS >= 3, "ring too shallow");
  static_assert(ACC0 + 2 * ACC_COLS <= 512, "tensor memory");
  static_assert(ATOM % 1024 == 0, "swizzled atoms need 1024-byte alignment");
};

// The work of round r (global index) of a launch.
struct Round {
  int unit, rr, jt, ob;
  bool ext;
  bool valid[2];
  int kb[2];     // main rounds: the K block of each slice
  int chunk[2];  // extension rounds: the 128-wide rank chunk of each slice
  int nk[2];     // 16-wide K steps of each slice
};

// Walks the rounds of a CTA's range in order without divisions: one division
// places it at the range's first round, then each advance is a few compares.
template <int NP>
struct RoundCursor {
  int unit, rr, jt, ob;
  int R, nmain, nkb, m_tiles, rank;
  __device__ __forceinline__ void init(long long r, int R_, int nmain_, int nkb_, int m_tiles_, int rank_) {
    R = R_;
    nmain = nmain_;
    nkb = nkb_;
    m_tiles = m_tiles_;
    rank = rank_;
    unit = (int)(r / R);
    rr = (int)(r - (long long)unit * R);
    jt = unit / m_tiles;
    ob = unit - jt * m_tiles;
  }
  __device__ __forceinline__ void advance() {
    if (++rr == R) {
      rr = 0;
      ++unit;
      if (++ob == m_tiles) {
        ob = 0;
        ++jt;
      }
    }
  }
  __device__ __forceinline__ Round get() const {
    Round o;
    o.unit = unit;
    o.rr = rr;
    o.jt = jt;
    o.ob = ob;
    o.ext = rr >= nmain;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (!o.ext) {
        o.kb[s] = NP == 2 ? rr : 2 * rr + s;
        o.valid[s] = o.kb[s] < nkb;
        o.chunk[s] = 0;
        o.nk[s] = 8;
      } else {
        const int e = rr - nmain;
        o.chunk[s] = NP == 2 ? e : 2 * e + s;
        o.valid[s] = o.chunk[s] * 128 < rank;
        o.kb[s] = 0;
        o.nk[s] = o.valid[s] ? (min(128, rank - o.chunk[s] * 128) + 15) / 16 : 0;
      }
    }
    return o;
  }
};

// First round of CTA c's range of `total` rounds over `g` CTAs.
__device__ __forceinline__ long long range_begin(long long total, int c, int g) { return total * c / g; }

// The CTA whose range holds round r.
__device__ __forceinline__ int cta_of(long long r, long long total, int g) {
  int c = (int)((r * g) / total);
  while (c + 1 < g && range_begin(total, c + 1, g) <= r) ++c;
  while (c > 0 && range_begin(total, c, g) > r) --c;
  return c;
}

// 16 codes of one tcgen05-layout word -> 8 fp16x2 of the exact q - z.
// nz[i] = -(1024 * 4^-i + z): the AND-OR places code field i above the fp16
// exponent of 1024 (value 1024 + 4^i q), the FMA by 4^-i removes the offset.
__device__ __forceinline__ void dq_qz_word(uint32_t w, const __half2 (&nz)[4], uint32_t *out) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 m[4] = {u32_as_h2(0x3C003C00u), u32_as_h2(0x34003400u), u32_as_h2(0x2C002C00u),
                        u32_as_h2(0x24002400u)};
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    const uint32_t v = hb ? (w >> 8) : w;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 x = u32_as_h2(and_or(v, 0x00030003u << (2 * i), kMagic));
      out[4 * hb + i] = h2_as_u32(__hfma2(x, m[i], nz[i]));
    }
  }
}

template <int NP, int BN, bool F8>
__global__ void __launch_bounds__(DQ_THREADS, 1) gemm_dq_kernel(const __grid_constant__ DqArgs P) {
  static_assert(!F8 || NP == 2, "fp8 mode: gate/up");
  using C = DqCfg<NP, BN>;
  constexpr int HC = BN / 2;  // accumulator columns per decode warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + C::NS;
  uint64_t *a_full = empty + C::NS;   // [2]
  uint64_t *mma_done = a_full + 2;    // [2]
  uint64_t *drain = mma_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  int *flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *fin = flag + 1;  // [BN]: combine, this CTA's slot was its token's last of the row block
  float *xbuf = reinterpret_cast<float *>(smem + C::XBUF_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto st_b = [&](int s) { return smem + s * C::STAGE; };
  auto st_codes = [&](int s, int sl) { return smem + s * C::STAGE + C::B_BYTES + sl * 4096; };
  auto st_sz = [&](int s, int sl) {
    return reinterpret_cast<const uint32_t *>(smem + s * C::STAGE + C::B_BYTES + C::CODES) + sl * 128;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DQ_DW);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&a_full[j], DQ_DW);
      mbar_init(&mma_done[j], 1);
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
  const int nkb = P.d_in / 128;
  const int G = P.d_in / P.group;
  const int nmain = NP == 2 ? nkb : (nkb + 1) / 2;
  const int n_ext = P.rank > 0 ? (NP == 2 ? (P.rank + 127) / 128 : (P.rank + 255) / 256) : 0;
  const int R = nmain + n_ext;  // rounds per unit
  const long long total = (long long)n_tiles * P.m_tiles * R;
  const long long r0 = range_begin(total, blockIdx.x, gridDim.x);
  const long long r1 = range_begin(total, blockIdx.x + 1, gridDim.x);
  const int nr = (int)(r1 - r0);
  bool ok = true;

  if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      int i = 0;
      RoundCursor<NP> cur;
      cur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
      for (; i < nr; ++i, cur.advance()) {
        const int s = i % C::NS;
        if (i >= C::NS && !(ok = mbar_wait(&empty[s], ((i / C::NS) - 1) & 1, P.status))) break;
        const Round rd = cur.get();
        const int4 t = P.tiles[rd.jt];
        const int grp = t.x, item0 = t.y;
        uint8_t *bs = st_b(s);
        if (!rd.ext) {
          uint32_t bytes = 0;
          int na = 0;
          for (int sl = 0; sl < 2; ++sl)
            if (rd.valid[sl]) {
              bytes += 4096 + 512;
              na += NP == 2 ? (sl == 0 ? 2 : 0) : 2;
            }
          mbar_arrive_expect_tx(&full[s], bytes + (uint32_t)na * C::ATOM);
          for (int sl = 0; sl < 2; ++sl) {
            if (!rd.valid[sl]) continue;
            const int p = NP == 2 ? sl : 0, kb = rd.kb[sl];
            const size_t blk = ((size_t)grp * P.m_tiles + rd.ob) * nkb + kb;
            bulk_g2s(st_codes(s, sl), reinterpret_cast<const uint8_t *>(P.codes[p]) + blk * 4096, 4096, &full[s]);
            const size_t zoff = (((size_t)grp * P.m_tiles + rd.ob) * G + (kb * 128) / P.group) * 128;
            bulk_g2s(const_cast<uint32_t *>(st_sz(s, sl)), P.sz[p] + zoff, 512, &full[s]);
            if (F8) {
              // the two e4m3 pieces of the 128 K of this block (one 128-byte box each)
              if (sl == 0)
                for (int pc = 0; pc < 2; ++pc)
                  tc::tma_load_2d(bs + pc * C::ATOM, &P.bmap, pc * P.d_in + kb * 128, item0, &full[s]);
            } else if (NP == 1 || sl == 0) {
              for (int a = 0; a < 2; ++a)
                tc::tma_load_2d(bs + (2 * sl + a) * C::ATOM, &P.bmap, kb * 128 + a * 64, item0, &full[s]);
            }
          }
        } else {
          int na = 0;
          for (int sl = 0; sl < 2; ++sl)
            if (rd.valid[sl]) na += (min(128, P.rank - rd.chunk[sl] * 128) + 63) / 64;
          mbar_arrive_expect_tx(&full[s], (uint32_t)na * C::ATOM);
          for (int sl = 0; sl < 2; ++sl) {
            if (!rd.valid[sl]) continue;
            const int p = NP == 2 ? sl : 0;
            const int len = min(128, P.rank - rd.chunk[sl] * 128);
            for (int a = 0; a * 64 < len; ++a)
              tc::tma_load_2d(bs + (2 * sl + a) * C::ATOM, F8 ? &P.bmap_ext : &P.bmap,
                              P.ext_col[p] + rd.chunk[sl] * 128 + a * 64, item0, &full[s]);
          }
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int j = i > C::NS ? i - C::NS : 0; j < i; ++j) mbar_wait(&full[j % C::NS], (j / C::NS) & 1, P.status);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = tc::idesc_f16(BN);
    RoundCursor<NP> cur;
    cur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    for (int i = 0; i < nr; ++i, cur.advance()) {
      const int as = i & 1;
      if (!(ok = mbar_wait(&a_full[as], (i >> 1) & 1, P.status))) break;
      tc::fence_after();
      const Round rd = cur.get();
      if (tc::elect_one()) {
        const uint64_t bd0 = tc::sdesc_sw128(smem_addr(st_b(i % C::NS)));
        const uint32_t a0 = tmem + as * 128, d0 = tmem + C::ACC0 + as * C::ACC_COLS;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          if (!rd.valid[sl]) continue;
          if (F8 && !rd.ext) {
            // e4m3: four K = 32 steps over 128 K; both pieces of B into the same accumulator
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
              for (int pc = 0; pc < 2; ++pc)
                tc::mma_ts_f8(d0 + sl * BN, a0 + sl * 64 + kk * 8,
                              bd0 + (uint64_t)((pc * C::ATOM + kk * 32) >> 4), idesc, (kk | pc) ? 1u : 0u);
            continue;
          }
          // B atoms of this slice: main rounds of a two-projection launch share atoms 0, 1
          const int atom0 = (NP == 2 && !rd.ext) ? 0 : 2 * sl;
          for (int kk = 0; kk < rd.nk[sl]; ++kk)
            tc::mma_ts(d0 + sl * BN, a0 + sl * 64 + kk * 8,
                       bd0 + (uint64_t)((((atom0 + kk / 4) * C::ATOM) + (kk % 4) * 32) >> 4), idesc, kk ? 1u : 0u);
        }
        tc::commit(&mma_done[as]);
      }
      __syncwarp();
    }
    // all issued MMAs have retired before TMEM is released
    if (tc::elect_one()) tc::commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, P.status);
  } else {
    // ============================================================ decode + epilogue
    const int dw = warp - 2;
    const int sub = dw >> 2;            // 0..3
    const int sl = sub >> 1;            // slice
    const int part = sub & 1;           // K half (decode) / column half (epilogue)
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tc::lane_base(warp);
    float acc[HC];
#pragma unroll
    for (int c = 0; c < HC; ++c) acc[c] = 0.f;
    float sc0 = 0.f, sc1 = 0.f;  // this row's scale of the warp's slice in the rounds of even / odd index
    bool v0 = false, v1 = false;  // the warp's slice was valid in the last round of even / odd index

    // ---- end of a unit's rounds in this CTA: combine the two slices, then
    // store the result (whole unit) or a piece (unit cut between CTAs)
    auto unit_end = [&](const Round &rd) -> void {
      const long long ustart = (long long)rd.unit * R, uend = ustart + R;
      const bool whole = ustart >= r0 && uend <= r1;
      const int4 t = P.tiles[rd.jt];
      const int item0 = t.y, nitems = t.z;
      const int o = rd.ob * 128 + row;
      named_sync(1, DQ_DW * 32);  // the previous unit's readers are done with xbuf
      if (sl == 1)
#pragma unroll
        for (int c = 0; c < HC; ++c) xbuf[(part * HC + c) * 128 + row] = acc[c];
      named_sync(1, DQ_DW * 32);
      if (sl == 0) {
        // the final result of item column n = part * HC + c: np = 2: silu(gate) * up * row scale (fp16),
        // np = 1: the sum of both slices (fp32)
        auto store = [&](int c, float g, float u) {
          const int n = part * HC + c;
          if (n >= nitems || o >= P.d_out) return;
          if (F8) {  // the activations were scaled by 2^e per item
            const float xs = __ldg(P.xs + item0 + n);
            g *= xs;
            u *= xs;
          }
          if (NP == 2 && P.epi == EPI_STORE2_F32) {
            reinterpret_cast<float *>(P.out)[(size_t)(item0 + n) * P.ldo + o] = g;
            reinterpret_cast<float *>(P.out2)[(size_t)(item0 + n) * P.ldo + o] = u;
          } else if (NP == 2) {
            const float rs = P.row_scale ? __ldg(P.row_scale + item0 + n) : 1.f;
            reinterpret_cast<__half *>(P.out)[(size_t)(item0 + n) * P.ldo + o] = half_checked(silu_f(g) * u * rs, P.status);
          } else {
            reinterpret_cast<float *>(P.out)[(size_t)(item0 + n) * P.ldo + o] = g;
          }
        };
        if (whole) {
#pragma unroll
          for (int c = 0; c < HC; ++c) {
            const float x = xbuf[(part * HC + c) * 128 + row];
            store(c, NP == 2 ? acc[c] : acc[c] + x, x);
          }
        } else {
          // piece of this CTA: slot 0 if the unit is the first of its range, else slot 1
          const int slot = (ustart <= r0) ? 0 : 1;
          float *pc = P.part + ((size_t)blockIdx.x * 2 + slot) * NP * BN * 128;
#pragma unroll
          for (int c = 0; c < HC; ++c) {
            const int col = part * HC + c;
            const float x = xbuf[col * 128 + row];
            pc[col * 128 + row] = NP == 2 ? acc[c] : acc[c] + x;
            if (NP == 2) pc[(BN + col) * 128 + row] = x;
          }
          __threadfence();
          named_sync(2, DQ_DW * 16);
          const int c_first = cta_of(ustart, total, gridDim.x), c_last = cta_of(uend - 1, total, gridDim.x);
          // CTAs with an empty range (fewer rounds than CTAs) leave no piece
          int pieces = 0;
          for (int cc = c_first; cc <= c_last; ++cc)
            pieces += range_begin(total, cc + 1, gridDim.x) > range_begin(total, cc, gridDim.x);
          if (dw == 0 && lane == 0) *flag = atomicAdd(&P.counters[rd.unit], 1) == pieces - 1;
          named_sync(2, DQ_DW * 16);
          if (*flag) {
            // the last piece in: sum all pieces of the unit in CTA order
            __threadfence();
#pragma unroll 1
            for (int c = 0; c < HC; ++c) {
              const int col = part * HC + c;
              float g = 0.f, u = 0.f;
              for (int cc = c_first; cc <= c_last; ++cc) {
                const long long b = range_begin(total, cc, gridDim.x);
                if (range_begin(total, cc + 1, gridDim.x) == b) continue;
                const int s2 = (b / R == rd.unit) ? 0 : 1;  // the unit is cta cc's first (slot 0) or last
                const float *q = P.part + ((size_t)cc * 2 + s2) * NP * BN * 128;
                g += __ldcg(q + col * 128 + row);
                if (NP == 2) u += __ldcg(q + (BN + col) * 128 + row);
              }
              store(c, g, u);
            }
            if (dw == 0 && lane == 0) P.counters[rd.unit] = 0;
          }
        }
        // weighted top-k combine: the slot weights are inside h, so the layer
        // output of a token is the plain sum of its slots' rows
        if (NP == 1 && P.combine && (whole || *flag)) {
          __threadfence();
          named_sync(2, DQ_DW * 16);
          const int tid = dw * 32 + lane;  // 0 .. 255 over the slice-0 warps
          if (tid < nitems) {
            const int tok = __ldg(P.slot_tok + item0 + tid);
            fin[tid] = atomicAdd(&P.tok_counters[tok * P.m_tiles + rd.ob], 1) == P.top_k - 1;
          }
          named_sync(2, DQ_DW * 16);
          __threadfence();
          const float *yb = reinterpret_cast<const float *>(P.out);
          for (int n = 0; n < nitems; ++n) {
            if (!fin[n]) continue;
            const int tok = __ldg(P.slot_tok + item0 + n);
            for (int r = tid; r < 128; r += DQ_DW * 16) {
              const int oo = rd.ob * 128 + r;
              if (oo >= P.d_out) continue;
              float y = P.yshared ? __ldg(P.yshared + (size_t)tok * P.ldo + oo) : 0.f;
              for (int j = 0; j < P.top_k; ++j)
                y += __ldcg(yb + (size_t)__ldg(P.slot_of_pair + tok * P.top_k + j) * P.ldo + oo);
              P.out_tok[(size_t)tok * P.ldo + oo] = __float2bfloat16_rn(y);
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < HC; ++c) acc[c] = 0.f;
    };

    // ---- fold round j's accumulator (slot j & 1) into registers; release its stage
    // (rounds are finished in order: fcur is at round j)
    RoundCursor<NP> fcur;
    fcur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    auto finish = [&](int j) -> bool {
      if (!mbar_wait(&mma_done[j & 1], (j >> 1) & 1, P.status)) return false;
      tc::fence_after();
      const float sc = (j & 1) ? sc1 : sc0;
      // tcgen05.ld is warp-collective: the decision is the warp's (its slice
      // was valid in round j), never a lane's (padding rows have scale 0)
      if ((j & 1) ? v1 : v0) {
        const uint32_t base = tmem + lane_addr + C::ACC0 + (j & 1) * C::ACC_COLS + sl * BN + part * HC;
#pragma unroll
        for (int c0 = 0; c0 < HC; c0 += 16) {
          uint32_t d[16];
          if constexpr (HC >= 16) {
            tc::ld16_nowait(base + c0, d);
          } else {
            float f[8];
            tc::ld8(base, f);
#pragma unroll
            for (int c = 0; c < 8; ++c) d[c] = __float_as_uint(f[c]);
          }
          tc::wait_ld();
#pragma unroll
          for (int c = 0; c < (HC < 16 ? HC : 16); ++c) acc[c0 + c] = fmaf(__uint_as_float(d[c]), sc, acc[c0 + c]);
        }
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[j % C::NS]);
      const Round rd = fcur.get();  // round j
      fcur.advance();
      if (rd.rr == R - 1 || j == nr - 1) unit_end(rd);
      return true;
    };

    RoundCursor<NP> cur;
    cur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    for (int i = 0; i < nr && ok; ++i, cur.advance()) {
      const int s = i % C::NS;
      if (!(ok = mbar_wait(&full[s], (i / C::NS) & 1, P.status))) break;
      // round i - 2: fold its accumulator; its A slot is then free for round i
      if (i >= 2 && !(ok = finish(i - 2))) break;
      const Round rd = cur.get();
      const bool mine = sl ? rd.valid[1] : rd.valid[0];
      const int chunk = sl ? rd.chunk[1] : rd.chunk[0];
      uint32_t v[32];
      float sc = 0.f;
      if (mine && !rd.ext) {
        // codes of this slice's K half: K slices 2 part and 2 part + 1 of the 4 x 32 layout
        const uint8_t *cb = st_codes(s, sl);
        uint32_t w[4];
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n"
                     : "=r"(w[0]), "=r"(w[1])
                     : "r"(smem_addr(cb + (2 * part) * 1024 + row * 8)));
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n"
                     : "=r"(w[2]), "=r"(w[3])
                     : "r"(smem_addr(cb + (2 * part + 1) * 1024 + row * 8)));
        const __half2 szw = u32_as_h2(st_sz(s, sl)[row]);
        if constexpr (F8) {
          // e4m3 (q - z) through a 4-entry byte table per zero point: one PRMT per 4 weights
          const int zi = (int)__high2float(szw);
          const uint32_t tab = zi == 0 ? 0x44403800u : zi == 1 ? 0x403800B8u : zi == 2 ? 0x3800B8C0u : 0x00B8C0C4u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t c0 = w[q] & 0x33333333u, c1 = (w[q] >> 2) & 0x33333333u;
            v[4 * q + 0] = __byte_perm(tab, 0, c0);
            v[4 * q + 1] = __byte_perm(tab, 0, c0 >> 16);
            v[4 * q + 2] = __byte_perm(tab, 0, c1);
            v[4 * q + 3] = __byte_perm(tab, 0, c1 >> 16);
          }
        } else {
          const __half2 z2 = __high2half2(szw);
          const __half2 nz[4] = {__hsub2(__float2half2_rn(-1024.f), z2), __hsub2(__float2half2_rn(-256.f), z2),
                                 __hsub2(__float2half2_rn(-64.f), z2), __hsub2(__float2half2_rn(-16.f), z2)};
#pragma unroll
          for (int q = 0; q < 4; ++q) dq_qz_word(w[q], nz, v + 8 * q);
        }
        sc = __low2float(szw);
      } else if (mine) {
        // rows of U_m: rank columns chunk * 128 + part * 64 ..
        const int4 t = P.tiles[rd.jt];
        const int p = NP == 2 ? sl : 0;
        const __half *ur =
            P.u[p] + (((size_t)P.u_blk[p][t.x] * P.m_tiles + rd.ob) * 128 + row) * P.rank + chunk * 128 + part * 64;
        const int kmax = P.rank - chunk * 128 - part * 64;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4 q4 = make_uint4(0, 0, 0, 0);
          if (j * 8 < kmax) q4 = __ldg(reinterpret_cast<const uint4 *>(ur + j * 8));
          v[4 * j + 0] = q4.x;
          v[4 * j + 1] = q4.y;
          v[4 * j + 2] = q4.z;
          v[4 * j + 3] = q4.w;
        }
        sc = 1.f;
      }
      if (mine) {
        if (F8 && !rd.ext) {
          tc::st16(tmem + lane_addr + (i & 1) * 128 + sl * 64 + part * 16, *reinterpret_cast<uint32_t(*)[16]>(v));
        } else {
          tc::st32(tmem + lane_addr + (i & 1) * 128 + sl * 64 + part * 32, v);
        }
        tc::wait_st();
      }
      if (i & 1) {
        sc1 = sc;
        v1 = mine;
      } else {
        sc0 = sc;
        v0 = mine;
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[i & 1]);
    }
    // the last two rounds' accumulators
    if (ok)
      for (int j = nr >= 2 ? nr - 2 : 0; j < nr && ok; ++j) ok = finish(j);
  }

  __syncwarp();
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

template <int NP, int BN, bool F8 = false>
cudaError_t launch_dq(const DqArgs &a, cudaStream_t stream) {
  using C = DqCfg<NP, BN>;
  auto kern = gemm_dq_kernel<NP, BN, F8>;
  static bool configured = false;  // one attribute call per instantiation and process
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const cudaError_t e = launch_pdl(kern, dim3(DQ_GRID), dim3(DQ_THREADS), C::SMEM, stream, a);
  if (e != cudaSuccess) return e;
  count_launches();
  return cudaGetLastError();
}

}  // namespace

int dq_grid() { return DQ_GRID; }

cudaError_t launch_gemm_dq(const DqArgs &a, int np, int bn, cudaStream_t stream) {
  if (a.m_tiles <= 0 || a.group % 128 != 0 || a.d_in % 128 != 0 || a.rank < 0 || a.rank > 256)
    return cudaErrorInvalidValue;
  if (a.f8) {
    if (np != 2) return cudaErrorInvalidValue;
    switch (bn) {
      case 16: return launch_dq<2, 16, true>(a, stream);
      case 32: return launch_dq<2, 32, true>(a, stream);
      case 64: return launch_dq<2, 64, true>(a, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (bn * 4 + np) {
    case 16 * 4 + 1: return launch_dq<1, 16>(a, stream);
    case 32 * 4 + 1: return launch_dq<1, 32>(a, stream);
    case 64 * 4 + 1: return launch_dq<1, 64>(a, stream);
    case 16 * 4 + 2: return launch_dq<2, 16>(a, stream);
    case 32 * 4 + 2: return launch_dq<2, 32>(a, stream);
    case 64 * 4 + 2: return launch_dq<2, 64>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tileq
