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
// Warp roles (6 warps): warp 0 producer (bulk copies of the codes and their
// (scale, zero) words in chunks of up to 8 K blocks per projection into a
// ring of chunk slots, 2-D TMA boxes of B per round into a ring of its own), warp 1 MMA
// issuer (the whole warp waits, one elected lane issues and commits), warps
// 2..5 decode and epilogue: warp w works on TMEM lane quadrant w % 4 (32
// weight rows) and both slices of every round (256 weights per thread and
// round, so that each barrier round amortises over enough decode work), with
// both slices' accumulators in its registers.
// Every wait is bounded and reports TILEQ_ERR_TIMEOUT.
#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int DQ_DW = 4;                      // decode / epilogue warps (one per TMEM lane quadrant)
constexpr int DQ_THREADS = (2 + DQ_DW) * 32;  // + producer + MMA issuer
constexpr int DQ_GRID = 148;                  // one CTA per SM

template <int NP, int BN>
struct DqCfg {
  static constexpr int ATOM = BN * 128;                // one 64-wide fp16 K atom of B: BN rows x 128 B
  static constexpr int B_BYTES = 4 * ATOM;             // up to four atoms per round
  // The codes stream from HBM in chunks of up to CB consecutive 128-wide K
  // blocks per projection (one bulk copy of up to 32 KB each, with the
  // (scale, zero) words of their groups): a few large copies in flight keep
  // the weight stream at the HBM rate, where one 4 KB copy per block does not.
  static constexpr int CB = 8;
  static constexpr int RPC = NP == 2 ? CB : CB / 2;     // main rounds per chunk
  static constexpr int CODE_SLOT = NP * CB * (4096 + 512);
  static constexpr int NB = 4;                         // activation ring (per round, from L2)
  static constexpr int NC_RAW = (210 * 1024 - NB * B_BYTES) / CODE_SLOT;
  static constexpr int NC = NC_RAW > 4 ? 4 : NC_RAW;   // code chunk ring
  static constexpr int CODE_OFF = NB * B_BYTES;
  static constexpr int BAR_OFF = CODE_OFF + NC * CODE_SLOT;
  static constexpr int SMEM = BAR_OFF + (2 * NB + 2 * NC + 5) * 8 + 16 + BN * 4 + 1024;  // + slack to align the base
  static constexpr int ACC_COLS = 2 * BN;             // one accumulator slot: two slices
  static constexpr int ACC0 = 256;                     // TMEM: A slots at 0 and 128, accumulators from 256
  static_assert(NC >= 2, "code ring too shallow");
  static_assert(ACC0 + 2 * ACC_COLS <= 512, "tensor memory");
  static_assert(ATOM % 1024 == 0, "swizzled atoms need 1024-byte alignment");
};

// Where a CTA's main rounds of one unit start new code chunks: chunks hold
// RPC consecutive main rounds from the first main round the CTA processes in
// the unit, up to its last one.  Producer and consumers step it the same way.
struct ChunkTrack {
  int rr_lo = 0, rr_hi = 0;  // main rounds [rr_lo, rr_hi) of the current unit in this CTA
  int n = 0;                 // chunks started so far
  template <int RPC>
  __device__ __forceinline__ void on_round(bool first_of_unit, int rr, int unit, int R, int nmain, long long r1) {
    if (first_of_unit) {
      rr_lo = rr;
      rr_hi = (int)min((long long)nmain, r1 - (long long)unit * R);
    }
  }
  template <int RPC>
  __device__ __forceinline__ bool starts(int rr) const { return rr < rr_hi && (rr - rr_lo) % RPC == 0; }
  template <int RPC>
  __device__ __forceinline__ bool ends(int rr) const {
    return rr < rr_hi && ((rr - rr_lo) % RPC == RPC - 1 || rr == rr_hi - 1);
  }
  template <int RPC>
  __device__ __forceinline__ int first_round(int rr) const { return rr - (rr - rr_lo) % RPC; }
  template <int RPC>
  __device__ __forceinline__ int last_round(int rr) const { return min(first_round<RPC>(rr) + RPC, rr_hi) - 1; }
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
  static_assert(BN == 16 || BN == 32, "16 or 32 items per tile");
  using C = DqCfg<NP, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *b_full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);  // [NB] activations of a round
  uint64_t *b_empty = b_full + C::NB;
  uint64_t *c_full = b_empty + C::NB;  // [NC] code chunks
  uint64_t *c_empty = c_full + C::NC;
  uint64_t *a_full = c_empty + C::NC;  // [2]
  uint64_t *mma_done = a_full + 2;    // [2]
  uint64_t *drain = mma_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  int *flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *fin_tok = flag + 1;  // [BN]: combine, this CTA's slot was its token's last of the row block

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto st_b = [&](int s) { return smem + s * C::B_BYTES; };
  // code chunk slot c: [projection][CB blocks of 4 KB], then [projection][CB groups of 128 (scale, zero) words]
  auto ch_codes = [&](int c, int p) { return smem + C::CODE_OFF + c * C::CODE_SLOT + p * C::CB * 4096; };
  auto ch_sz = [&](int c, int p) {
    return reinterpret_cast<uint32_t *>(smem + C::CODE_OFF + c * C::CODE_SLOT + NP * C::CB * 4096) + p * C::CB * 128;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], DQ_DW);
    }
    for (int c = 0; c < C::NC; ++c) {
      mbar_init(&c_full[c], 1);
      mbar_init(&c_empty[c], DQ_DW);
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
      ChunkTrack ck;
      int cur_jt = -1;
      int4 cur_tile = make_int4(0, 0, 0, 0);
      for (; i < nr; ++i, cur.advance()) {
        const Round rd = cur.get();
        ck.on_round<C::RPC>(i == 0 || rd.rr == 0, rd.rr, rd.unit, R, nmain, r1);
        if (rd.jt != cur_jt) {  // the tile changes with the unit only
          cur_jt = rd.jt;
          cur_tile = P.tiles[rd.jt];
        }
        const int grp = cur_tile.x, item0 = cur_tile.y;
        if (!rd.ext && ck.starts<C::RPC>(rd.rr)) {
          // the next code chunk: rounds first .. last of this unit
          const int c = ck.n % C::NC;
          if (ck.n >= C::NC && !(ok = mbar_wait(&c_empty[c], ((ck.n / C::NC) - 1) & 1, P.status))) break;
          const int r_a = rd.rr, r_b = ck.last_round<C::RPC>(rd.rr) + 1;
          const int kb_a = NP == 2 ? r_a : 2 * r_a, kb_b = NP == 2 ? r_b : min(nkb, 2 * r_b);
          const int g_a = (kb_a * 128) / P.group, g_b = ((kb_b - 1) * 128) / P.group;
          const uint32_t cbytes = (uint32_t)(kb_b - kb_a) * 4096, zbytes = (uint32_t)(g_b - g_a + 1) * 512;
          mbar_arrive_expect_tx(&c_full[c], NP * (cbytes + zbytes));
          for (int p = 0; p < NP; ++p) {
            const size_t blk = ((size_t)grp * P.m_tiles + rd.ob) * nkb + kb_a;
            bulk_g2s(ch_codes(c, p), reinterpret_cast<const uint8_t *>(P.codes[p]) + blk * 4096, cbytes, &c_full[c]);
            const size_t zoff = (((size_t)grp * P.m_tiles + rd.ob) * G + g_a) * 128;
            bulk_g2s(ch_sz(c, p), P.sz[p] + zoff, zbytes, &c_full[c]);
          }
          ++ck.n;
        }
        // the round's activation tile
        const int s = i % C::NB;
        if (i >= C::NB && !(ok = mbar_wait(&b_empty[s], ((i / C::NB) - 1) & 1, P.status))) break;
        uint8_t *bs = st_b(s);
        if (!rd.ext) {
          int na = 0;
          for (int sl = 0; sl < 2; ++sl)
            if (rd.valid[sl]) na += (NP == 2 || F8) ? (sl == 0 ? 2 : 0) : 2;
          mbar_arrive_expect_tx(&b_full[s], (uint32_t)na * C::ATOM);
          for (int sl = 0; sl < 2; ++sl) {
            if (!rd.valid[sl]) continue;
            const int kb = rd.kb[sl];
            if (F8) {
              // the two e4m3 pieces of the 128 K of this block (one 128-byte box each)
              if (sl == 0)
                for (int pc = 0; pc < 2; ++pc)
                  tc::tma_load_2d(bs + pc * C::ATOM, &P.bmap, pc * P.d_in + kb * 128, item0, &b_full[s]);
            } else if (NP == 1 || sl == 0) {
              for (int a = 0; a < 2; ++a)
                tc::tma_load_2d(bs + (2 * sl + a) * C::ATOM, &P.bmap, kb * 128 + a * 64, item0, &b_full[s]);
            }
          }
        } else {
          int na = 0;
          for (int sl = 0; sl < 2; ++sl)
            if (rd.valid[sl]) na += (min(128, P.rank - rd.chunk[sl] * 128) + 63) / 64;
          mbar_arrive_expect_tx(&b_full[s], (uint32_t)na * C::ATOM);
          for (int sl = 0; sl < 2; ++sl) {
            if (!rd.valid[sl]) continue;
            const int p = NP == 2 ? sl : 0;
            const int len = min(128, P.rank - rd.chunk[sl] * 128);
            for (int a = 0; a * 64 < len; ++a)
              tc::tma_load_2d(bs + (2 * sl + a) * C::ATOM, F8 ? &P.bmap_ext : &P.bmap,
                              P.ext_col[p] + rd.chunk[sl] * 128 + a * 64, item0, &b_full[s]);
          }
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int j = i > C::NB ? i - C::NB : 0; j < i; ++j) mbar_wait(&b_full[j % C::NB], (j / C::NB) & 1, P.status);
      for (int j = ck.n > C::NC ? ck.n - C::NC : 0; j < ck.n; ++j)
        mbar_wait(&c_full[j % C::NC], (j / C::NC) & 1, P.status);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = tc::idesc_f16(BN);
    RoundCursor<NP> cur;
    cur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    for (int i = 0; i < nr; ++i, cur.advance()) {
      const int as = i & 1;
      if (!(ok = mbar_wait(&a_full[as], (i >> 1) & 1, P.status))) break;
      if (!(ok = mbar_wait(&b_full[i % C::NB], (i / C::NB) & 1, P.status))) break;
      tc::fence_after();
      const Round rd = cur.get();
      if (tc::elect_one()) {
        const uint64_t bd0 = tc::sdesc_sw128(smem_addr(st_b(i % C::NB)));
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
    // One warp per TMEM lane quadrant (32 weight rows): it decodes both slices
    // of every round (256 weights per thread) and holds both accumulators in
    // registers, so a unit's two slices meet in the same thread.
    const int dw = warp - 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tc::lane_base(warp);
    float acc0[BN], acc1[BN];  // np = 2: gate, up; np = 1: the two slices' partial sums
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      acc0[c] = 0.f;
      acc1[c] = 0.f;
    }
    // per round parity (e: even index, o: odd): this row's scale of each slice and whether the slice was valid
    float sce0 = 0.f, sce1 = 0.f, sco0 = 0.f, sco1 = 0.f;
    bool vde0 = false, vde1 = false, vdo0 = false, vdo1 = false;

    // ---- end of a unit's rounds in this CTA: store the result (whole unit) or
    // a piece (unit cut between CTAs; the CTA finishing last sums them)
    auto unit_end = [&](const Round &rd) -> void {
      const long long ustart = (long long)rd.unit * R, uend = ustart + R;
      const bool whole = ustart >= r0 && uend <= r1;
      const int4 t = P.tiles[rd.jt];
      const int item0 = t.y, nitems = t.z;
      const int o = rd.ob * 128 + row;
      // the final result of item column n: np = 2: silu(gate) * up * row scale (fp16) or both in
      // fp32; np = 1: the sum of both slices (fp32)
      auto store = [&](int n, float g, float u) {
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
      bool fin = whole;
      if (whole) {
#pragma unroll
        for (int c = 0; c < BN; ++c) store(c, NP == 2 ? acc0[c] : acc0[c] + acc1[c], acc1[c]);
      } else {
        // piece of this CTA: slot 0 if the unit is the first of its range, else slot 1
        const int slot = (ustart <= r0) ? 0 : 1;
        float *pc = P.part + ((size_t)blockIdx.x * 2 + slot) * NP * BN * 128;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          pc[c * 128 + row] = NP == 2 ? acc0[c] : acc0[c] + acc1[c];
          if (NP == 2) pc[(BN + c) * 128 + row] = acc1[c];
        }
        __threadfence();
        named_sync(1, DQ_DW * 32);
        const int c_first = cta_of(ustart, total, gridDim.x), c_last = cta_of(uend - 1, total, gridDim.x);
        // CTAs with an empty range (fewer rounds than CTAs) leave no piece
        int pieces = 0;
        for (int cc = c_first; cc <= c_last; ++cc)
          pieces += range_begin(total, cc + 1, gridDim.x) > range_begin(total, cc, gridDim.x);
        if (dw == 0 && lane == 0) *flag = atomicAdd(&P.counters[rd.unit], 1) == pieces - 1;
        named_sync(1, DQ_DW * 32);
        fin = *flag != 0;
        if (fin) {
          // the last piece in: sum all pieces of the unit in CTA order
          __threadfence();
#pragma unroll 1
          for (int c = 0; c < BN; ++c) {
            float g = 0.f, u = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const long long b = range_begin(total, cc, gridDim.x);
              if (range_begin(total, cc + 1, gridDim.x) == b) continue;
              const int s2 = (b / R == rd.unit) ? 0 : 1;  // the unit is cta cc's first (slot 0) or last
              const float *q = P.part + ((size_t)cc * 2 + s2) * NP * BN * 128;
              g += __ldcg(q + c * 128 + row);
              if (NP == 2) u += __ldcg(q + (BN + c) * 128 + row);
            }
            store(c, g, u);
          }
          if (dw == 0 && lane == 0) P.counters[rd.unit] = 0;
        }
      }
      // weighted top-k combine: the slot weights are inside h, so the layer
      // output of a token is the plain sum of its slots' rows
      if (NP == 1 && P.combine && fin) {
        __threadfence();
        named_sync(1, DQ_DW * 32);
        const int tid = dw * 32 + lane;  // 0 .. 127
        if (tid < nitems) {
          const int tok = __ldg(P.slot_tok + item0 + tid);
          fin_tok[tid] = atomicAdd(&P.tok_counters[tok * P.m_tiles + rd.ob], 1) == P.top_k - 1;
        }
        named_sync(1, DQ_DW * 32);
        __threadfence();
        const float *yb = reinterpret_cast<const float *>(P.out);
        for (int n = 0; n < nitems; ++n) {
          if (!fin_tok[n]) continue;
          const int tok = __ldg(P.slot_tok + item0 + n);
          const int oo = rd.ob * 128 + tid;
          if (oo >= P.d_out) continue;
          float y = P.yshared ? __ldg(P.yshared + (size_t)tok * P.ldo + oo) : 0.f;
          for (int j = 0; j < P.top_k; ++j)
            y += __ldcg(yb + (size_t)__ldg(P.slot_of_pair + tok * P.top_k + j) * P.ldo + oo);
          P.out_tok[(size_t)tok * P.ldo + oo] = __float2bfloat16_rn(y);
        }
        named_sync(1, DQ_DW * 32);  // fin_tok is reused by the next unit
      }
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        acc0[c] = 0.f;
        acc1[c] = 0.f;
      }
    };

    // fold one slice's accumulator (BN columns at TMEM column base) into acc
    auto fold = [&](uint32_t base, float s, float (&acc)[BN]) {
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t d[16];
        tc::ld16_nowait(base + c0, d);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c0 + c] = fmaf(__uint_as_float(d[c]), s, acc[c0 + c]);
      }
    };

    // ---- fold round j's accumulators (slot j & 1) into registers; release its stage
    // (rounds are finished in order: fcur is at round j)
    RoundCursor<NP> fcur;
    fcur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    auto finish = [&](int j) -> bool {
      if (!mbar_wait(&mma_done[j & 1], (j >> 1) & 1, P.status)) return false;
      tc::fence_after();
      const uint32_t base = tmem + lane_addr + C::ACC0 + (j & 1) * C::ACC_COLS;
      // tcgen05.ld is warp-collective: the decision is the warp's (the slice
      // was valid in round j), never a lane's (padding rows have scale 0)
      const bool odd = j & 1;
      if (odd ? vdo0 : vde0) fold(base, odd ? sco0 : sce0, acc0);
      if (odd ? vdo1 : vde1) fold(base + BN, odd ? sco1 : sce1, acc1);
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_empty[j % C::NB]);
      const Round rd = fcur.get();  // round j
      fcur.advance();
      if (rd.rr == R - 1 || j == nr - 1) unit_end(rd);
      return true;
    };

    // ---- one slice of round i into the A slot: decode (main) or U_m rows (extension)
    auto load_slice = [&](const Round &rd, int c, int kb_a, int g_a, int sl, int i, float &scale) {
      const uint32_t acol = tmem + lane_addr + (i & 1) * 128 + sl * 64;
      if (!rd.ext) {
        const int p = NP == 2 ? sl : 0, kb = sl ? rd.kb[1] : rd.kb[0];
        const uint8_t *cb = ch_codes(c, p) + (kb - kb_a) * 4096;
        const __half2 szw = u32_as_h2(ch_sz(c, p)[((kb * 128) / P.group - g_a) * 128 + row]);
        scale = __low2float(szw);
        if constexpr (F8) {
          // e4m3 (q - z) through a 4-entry byte table per zero point: one PRMT per 4 weights
          const int zi = (int)__high2float(szw);
          const uint32_t tab = zi == 0 ? 0x44403800u : zi == 1 ? 0x403800B8u : zi == 2 ? 0x3800B8C0u : 0x00B8C0C4u;
          uint32_t v[32];
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {  // the four K slices of 32 (two words of 16 codes each)
            uint32_t w0, w1;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(w0), "=r"(w1) : "r"(smem_addr(cb + ks * 1024 + row * 8)));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t w = h ? w1 : w0;
              const uint32_t c0 = w & 0x33333333u, c1 = (w >> 2) & 0x33333333u;
              uint32_t *o = v + 8 * ks + 4 * h;
              o[0] = __byte_perm(tab, 0, c0);
              o[1] = __byte_perm(tab, 0, c0 >> 16);
              o[2] = __byte_perm(tab, 0, c1);
              o[3] = __byte_perm(tab, 0, c1 >> 16);
            }
          }
          tc::st32(acol, v);
        } else {
          const __half2 z2 = __high2half2(szw);
          const __half2 nz[4] = {__hsub2(__float2half2_rn(-1024.f), z2), __hsub2(__float2half2_rn(-256.f), z2),
                                 __hsub2(__float2half2_rn(-64.f), z2), __hsub2(__float2half2_rn(-16.f), z2)};
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {  // K halves of 64: 32 TMEM columns each
            uint32_t v[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t w0, w1;
              asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n"
                           : "=r"(w0), "=r"(w1)
                           : "r"(smem_addr(cb + (2 * hk + q) * 1024 + row * 8)));
              dq_qz_word(w0, nz, v + 16 * q);
              dq_qz_word(w1, nz, v + 16 * q + 8);
            }
            tc::st32(acol + hk * 32, v);
          }
        }
      } else {
        // rows of U_m: rank columns chunk * 128 ..
        const int4 t = P.tiles[rd.jt];
        const int p = NP == 2 ? sl : 0;
        const int chunk = sl ? rd.chunk[1] : rd.chunk[0];
        const __half *ur = P.u[p] + (((size_t)P.u_blk[p][t.x] * P.m_tiles + rd.ob) * 128 + row) * P.rank + chunk * 128;
        const int kmax = P.rank - chunk * 128;
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {
          uint32_t v[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 q4 = make_uint4(0, 0, 0, 0);
            if (hk * 64 + j * 8 < kmax) q4 = __ldg(reinterpret_cast<const uint4 *>(ur + hk * 64 + j * 8));
            v[4 * j + 0] = q4.x;
            v[4 * j + 1] = q4.y;
            v[4 * j + 2] = q4.z;
            v[4 * j + 3] = q4.w;
          }
          tc::st32(acol + hk * 32, v);
        }
        scale = 1.f;
      }
    };

    RoundCursor<NP> cur;
    cur.init(r0, R, nmain, nkb, P.m_tiles, P.rank);
    ChunkTrack ck;
    int c = 0, kb_a = 0, g_a = 0;  // the current code chunk: ring slot, first block, first group
    for (int i = 0; i < nr && ok; ++i, cur.advance()) {
      const Round rd = cur.get();
      ck.on_round<C::RPC>(i == 0 || rd.rr == 0, rd.rr, rd.unit, R, nmain, r1);
      if (!rd.ext && ck.starts<C::RPC>(rd.rr)) {
        c = ck.n % C::NC;
        kb_a = NP == 2 ? rd.rr : 2 * rd.rr;
        g_a = (kb_a * 128) / P.group;
        if (!(ok = mbar_wait(&c_full[c], (ck.n / C::NC) & 1, P.status))) break;
        ++ck.n;
      }
      // round i - 2: fold its accumulators; its A slot is then free for round i
      if (i >= 2 && !(ok = finish(i - 2))) break;
      float s0 = 0.f, s1 = 0.f;
      if (rd.valid[0]) load_slice(rd, c, kb_a, g_a, 0, i, s0);
      if (rd.valid[1]) load_slice(rd, c, kb_a, g_a, 1, i, s1);
      // the chunk's codes are decoded: the producer may refill its slot
      if (!rd.ext && ck.ends<C::RPC>(rd.rr)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&c_empty[c]);
      }
      tc::wait_st();
      if (i & 1) {
        sco0 = s0;
        sco1 = s1;
        vdo0 = rd.valid[0];
        vdo1 = rd.valid[1];
      } else {
        sce0 = s0;
        sce1 = s1;
        vde0 = rd.valid[0];
        vde1 = rd.valid[1];
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
      default: return cudaErrorInvalidValue;
    }
  }
  switch (bn * 4 + np) {
    case 16 * 4 + 1: return launch_dq<1, 16>(a, stream);
    case 32 * 4 + 1: return launch_dq<1, 32>(a, stream);
    case 16 * 4 + 2: return launch_dq<2, 16>(a, stream);
    case 32 * 4 + 2: return launch_dq<2, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tileq
