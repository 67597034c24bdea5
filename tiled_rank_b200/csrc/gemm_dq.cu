// Residual GEMM of the decode regime (a handful of tokens per expert) on the
// 5th-generation tensor cores, for the TileQ forward (opt-in: the planner
// uses warp-level MMA for these tiles unless TILEQ_DECODE_TC=1):
//
//   out[item][o] = epi( sum_k s*(q - z)[o][k] * B[item][k]  +  sum_i U_m[o][i] * B[item][ext + i] )
//
//   * the A operand is the exact q - z of each 2-bit code, written to tensor
//     memory: in fp8 mode (gate/up) as e4m3 through a 4-byte table per zero
//     point (one PRMT per 4 weights), with B as two e4m3 pieces of the
//     activations; otherwise in fp16 (one AND-OR with the fp16 exponent of
//     1024 and one FMA per pair of weights).  TS-form tcgen05.mma, M = 128
//     weight rows, N = 16 or 32 items;
//   * every 128-wide K block (one scale group, or part of one) accumulates
//     into its own fp32 accumulator in tensor memory; the fold warps add it
//     into registers with the group scale (w = s*(q - z) is never rounded);
//   * a round = two slices of 128 K: gate and up of one K block (np = 2) or
//     two consecutive K blocks of one projection (np = 1);
//   * stream-K: the (tile, row block, round) space is cut into gridDim.x equal
//     contiguous ranges, one per CTA (one CTA per SM).  A (tile, row block)
//     unit cut between CTAs leaves fp32 pieces that the CTA finishing last
//     sums in CTA order (deterministic), so every SM streams the same number
//     of weight bytes whatever the routing.
// The low-rank term is a K extension: after a unit's residual rounds, the A
// slot holds rows of the grid row's U_m (fp16, read from global memory) and B
// the matching z (or a) columns of the item rows, with scale 1.
//
// Warp roles (14 warps), each a pipeline stage with its own ring:
//   warp 0       producer: per chunk (two rounds of one kind of a unit) the
//                codes, their (scale, zero) words and the rounds' activation
//                tiles into one ring slot, one copy per lane;
//   warp 1       MMA issuer: waits for a round's chunk, operand slot and
//                accumulator slot; one elected lane issues and commits to the
//                operand slot, the accumulator slot and, after the chunk's
//                last round, the chunk;
//   warps 2..9   decode: two warps per TMEM lane quadrant (32 weight rows), one
//                per slice, write every round into its operand slot and hand
//                the rows' group scales to the fold warps;
//   warps 10..13 fold + epilogue: one warp per lane quadrant folds every
//                round's accumulators with the group scales and stores units.
// A table of every round's descriptor is built before the pipeline starts.
// Every wait is bounded and reports TILEQ_ERR_TIMEOUT.
#include "kernels.cuh"
#include "tc.cuh"

namespace tileq {

namespace {

constexpr int DQ_DEC = 8;                             // decode warps: two per TMEM lane quadrant (one per slice)
constexpr int DQ_FW = 4;                              // fold / epilogue warps: one per lane quadrant
constexpr int DQ_THREADS = (2 + DQ_DEC + DQ_FW) * 32;  // + producer + MMA issuer
constexpr int DQ_GRID = 148;                          // one CTA per SM
constexpr int DQ_MAX_ROUNDS = 1024;                   // rounds of one CTA (its descriptor table)

template <int NP, int BN, bool F8>
struct DqCfg {
  static constexpr int ATOM = BN * 128;  // one 128-byte-wide K atom of B: BN rows x 128 B
  // B atoms per round: fp8 mode two (the two e4m3 pieces of 128 K, or one
  // 64-wide fp16 extension atom per slice), else up to four
  static constexpr int B_ROUND = (F8 ? 2 : 4) * ATOM;
  // A chunk is RPC consecutive rounds of one kind (residual or extension) of
  // a unit: the codes of CB K blocks per projection, their (scale, zero)
  // words and the rounds' activation tiles, loaded together by one warp
  // instruction with one copy per lane.  (A single thread completes about one
  // bulk copy per memory latency, so the copies of a chunk go out in parallel.)
  static constexpr int CB = NP == 2 ? 2 : 4;
  static constexpr int RPC = 2;
  static constexpr int SZ_OFF = NP * CB * 4096;
  static constexpr int B_OFF = (SZ_OFF + NP * CB * 512 + 1023) / 1024 * 1024;
  static constexpr int SLOT = B_OFF + RPC * B_ROUND;
  static constexpr int NC_RAW = 196 * 1024 / SLOT;
  static constexpr int NC = NC_RAW > 8 ? 8 : NC_RAW;  // chunk ring
  static constexpr int MAX_KB = 256;                  // K blocks of 128 (d_in up to 32768)
  static constexpr int GIDX_OFF = NC * SLOT;          // [MAX_KB] scale group of each K block
  static constexpr int TAB_OFF = GIDX_OFF + MAX_KB * 4;  // [DQ_MAX_ROUNDS] round descriptors
  // the decode warps hand each row's group scale to the fold warps through a
  // ring of NS rounds, so that a chunk is free once decoded
  static constexpr int NS = 16;
  static constexpr int SBUF_OFF = TAB_OFF + DQ_MAX_ROUNDS * 8;  // [NS][2 slices][128 rows] fp16
  static constexpr int BAR_OFF = SBUF_OFF + NS * 2 * 128 * 2;
  // Tensor memory: NA operand slots of one round (two slices: 128 K of e4m3
  // or 64 fp16 in fp8 mode, 128 fp16 otherwise), then NT accumulator slots of
  // one round (two slices of BN columns).
  static constexpr int EXT_W = F8 ? 64 : 128;  // rank columns of a slice in an extension round
  static constexpr int NT = 4;
  static constexpr int ACC_COLS = 2 * BN;
  static constexpr int A_COLS = F8 ? 64 : 128;
  static constexpr int SCOLS = A_COLS / 2;
  static constexpr int NA_RAW = (512 - NT * ACC_COLS) / A_COLS;
  static constexpr int NA = NA_RAW > 4 ? 4 : NA_RAW;
  static constexpr int ACC0 = NA * A_COLS;
  static constexpr int NBAR = 2 * NC + 2 * NA + 2 * NT + NS + 1;
  static constexpr int SMEM = BAR_OFF + NBAR * 8 + 16 + BN * 4 + 1024;  // + slack to align the base
  static_assert(NC >= 3, "chunk ring too shallow");
  static_assert(2 * NP + RPC * 4 <= 32, "one copy per lane");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NA >= 2, "operand ring too shallow");
  static_assert(NS > NA + NT, "scale ring: the decode runs at most NA + NT rounds ahead of the fold");
  static_assert(ACC0 + NT * ACC_COLS <= 512, "tensor memory");
  static_assert(ATOM % 1024 == 0 && B_OFF % 1024 == 0 && SLOT % 1024 == 0, "swizzled atoms need 1024-byte alignment");
};

// Bounded wait that lets the hardware suspend the warp until the phase
// completes (or the hint elapses) instead of spinning on the issue slots the
// decoding warps need.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, int *status) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(0x100000u)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const long long t0 = clock64();
  while (!try_once()) {
    if (clock64() - t0 > kWaitLimitCycles) {
      set_status(status, TILEQ_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Non-blocking probe of a phase (the result is consumed later, so its latency
// overlaps other work).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-round descriptor, one table per CTA built before the pipeline starts
// (x: flags below; y: unit << 9 | round within the unit), so that no warp
// walks the round space or waits for a descriptor.
enum : uint32_t {
  RD_EXT = 1u,         // U_m extension round
  RD_V0 = 2u,          // slice 0 valid
  RD_V1 = 4u,          // slice 1 valid
  RD_CSTART = 8u,      // first round of a code chunk
  RD_CEND = 16u,       // last round of a code chunk
  RD_UEND = 32u,       // last round of the unit in this CTA
  // bits 8..10 chunk ring slot, bit 11 its fill parity; bits 12..15 / 16..19:
  // 16-wide K steps of each slice (extension); bits 20..23: K block of each
  // slice within the chunk; bits 24..27: scale group of each slice within the
  // chunk; bits 28..29 / 30..31: rank chunk of each slice (extension)
};
__device__ __forceinline__ uint32_t rd_field(uint32_t f, int lo, int bits) { return (f >> lo) & ((1u << bits) - 1u); }

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
  using C = DqCfg<NP, BN, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *c_full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);  // [NC] chunks
  uint64_t *c_empty = c_full + C::NC;
  uint64_t *a_full = c_empty + C::NC;  // [NA] operand slots
  uint64_t *a_free = a_full + C::NA;
  uint64_t *acc_full = a_free + C::NA;  // [NT] accumulator slots
  uint64_t *acc_free = acc_full + C::NT;
  uint64_t *s_full = acc_free + C::NT;  // [NS] scales of a round written
  uint64_t *drain = s_full + C::NS;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  int *flag = reinterpret_cast<int *>(tmem_slot + 1);
  int *fin_tok = flag + 1;  // [BN]: combine, this CTA's slot was its token's last of the row block
  int *gidx = reinterpret_cast<int *>(smem + C::GIDX_OFF);
  int2 *tab = reinterpret_cast<int2 *>(smem + C::TAB_OFF);
  unsigned short *sbuf = reinterpret_cast<unsigned short *>(smem + C::SBUF_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // chunk slot c: [projection][CB blocks of 4 KB] codes, [projection][CB groups of 128] (scale, zero)
  // words, then the activation tiles of its rounds
  auto ch_codes = [&](int c, int p) { return smem + c * C::SLOT + p * C::CB * 4096; };
  auto ch_sz = [&](int c, int p) { return reinterpret_cast<uint32_t *>(smem + c * C::SLOT + C::SZ_OFF) + p * C::CB * 128; };
  auto ch_b = [&](int c, int pos) { return smem + c * C::SLOT + C::B_OFF + pos * C::B_ROUND; };

  const int nkb = P.d_in / 128;
  const int nmain = NP == 2 ? nkb : (nkb + 1) / 2;
  const int n_ext = P.rank > 0 ? (NP == 2 ? (P.rank + C::EXT_W - 1) / C::EXT_W : (P.rank + 255) / 256) : 0;
  const int R = nmain + n_ext;  // rounds per unit

  if (threadIdx.x == 0) {
    for (int c = 0; c < C::NC; ++c) {
      mbar_init(&c_full[c], 1);
      mbar_init(&c_empty[c], DQ_DEC + 1);  // the decode warps (codes) and the MMA warp (activations)
    }
    for (int j = 0; j < C::NA; ++j) {
      mbar_init(&a_full[j], DQ_DEC);
      mbar_init(&a_free[j], 1);
    }
    for (int j = 0; j < C::NT; ++j) {
      mbar_init(&acc_full[j], 1);
      mbar_init(&acc_free[j], DQ_FW);
    }
    for (int j = 0; j < C::NS; ++j) mbar_init(&s_full[j], DQ_DEC);
    mbar_init(drain, 1);
    *flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::alloc(tmem_slot, 512);
    tc::relinquish();
  }
  for (int k = threadIdx.x; k < nkb; k += blockDim.x) gidx[k] = (k * 128) / P.group;
  // the prologue above (barriers, TMEM, group table) overlaps the previous kernel's tail
  pdl_wait_and_release();

  const int n_tiles = *P.tile_count;
  const long long total = (long long)n_tiles * P.m_tiles * R;
  const long long r0 = range_begin(total, blockIdx.x, gridDim.x);
  const long long r1 = range_begin(total, blockIdx.x + 1, gridDim.x);
  const int nr_all = (int)(r1 - r0);
  // (the host keeps every CTA within the table; a launch outside it does nothing but report)
  const int nr = nr_all <= DQ_MAX_ROUNDS ? nr_all : 0;
  if (nr_all > DQ_MAX_ROUNDS && threadIdx.x == 0) set_status(P.status, TILEQ_ERR_UNSUPPORTED);

  // ---- the round table.  A chunk holds up to RPC consecutive rounds of one
  // kind (residual, then extension) of a unit, counted from the first round of
  // that kind this CTA processes in the unit.  Units strictly inside the range
  // are whole, so the chunks before a unit have a closed form.
  {
    const long long u0 = r0 / R;
    const int rr0 = (int)(r0 - u0 * R);
    auto cdv = [](int a, int b) { return (a + b - 1) / b; };
    // rounds [lo, hi) of unit u in this CTA, split into residual and extension runs
    auto lo_of = [&](long long u) { return u == u0 ? rr0 : 0; };
    auto hi_of = [&](long long u) { return (int)min((long long)R, r1 - u * R); };
    auto n_main_ch = [&](long long u) {
      const int lo = lo_of(u), hi = min(hi_of(u), nmain);
      return hi > lo ? cdv(hi - lo, C::RPC) : 0;
    };
    auto n_ext_ch = [&](long long u) {
      const int lo = max(lo_of(u), nmain), hi = hi_of(u);
      return hi > lo ? cdv(hi - lo, C::RPC) : 0;
    };
    const int nch0 = n_main_ch(u0) + n_ext_ch(u0);
    const int nch_full = cdv(nmain, C::RPC) + cdv(n_ext, C::RPC);
    for (int i = threadIdx.x; i < nr; i += blockDim.x) {
      const long long r = r0 + i;
      const long long unit = r / R;
      const int rr = (int)(r - unit * R);
      const int lo = lo_of(unit), hi = hi_of(unit);
      const int before = unit == u0 ? 0 : nch0 + (int)(unit - u0 - 1) * nch_full;
      uint32_t f = (rr == R - 1 || i == nr - 1) ? RD_UEND : 0u;
      int idx, pos, last;
      if (rr < nmain) {
        idx = before + (rr - lo) / C::RPC;
        pos = (rr - lo) % C::RPC;
        last = min(hi, nmain) - 1;
        const int kb_a = NP == 2 ? rr - pos : 2 * (rr - pos);
        const int kb0 = NP == 2 ? rr : 2 * rr, kb1 = NP == 2 ? rr : 2 * rr + 1;
        const int ga = (kb_a * 128) / P.group;
        f |= RD_V0;
        f |= (uint32_t)(kb0 - kb_a) << 20 | (uint32_t)((kb0 * 128) / P.group - ga) << 24;
        if (kb1 < nkb) f |= RD_V1 | (uint32_t)(kb1 - kb_a) << 22 | (uint32_t)((kb1 * 128) / P.group - ga) << 26;
      } else {
        const int lo_e = max(lo, nmain);
        idx = before + n_main_ch(unit) + (rr - lo_e) / C::RPC;
        pos = (rr - lo_e) % C::RPC;
        last = hi - 1;
        const int e = rr - nmain;
        f |= RD_EXT;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int ch = NP == 2 ? e : 2 * e + sl;
          if (ch * C::EXT_W < P.rank) {
            f |= (sl ? RD_V1 : RD_V0) | (uint32_t)((min(C::EXT_W, P.rank - ch * C::EXT_W) + 15) / 16) << (sl ? 16 : 12) |
                 (uint32_t)ch << (sl ? 30 : 28);
          }
        }
      }
      f |= (pos == 0 ? RD_CSTART : 0u) | (pos == C::RPC - 1 || rr == last ? RD_CEND : 0u) | (uint32_t)pos << 6;
      f |= (uint32_t)(idx % C::NC) << 8 | (uint32_t)((idx / C::NC) & 1) << 11;
      tab[i] = make_int2((int)f, (int)(unit << 9 | rr));
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ============================================================ producer
    // The whole warp walks the chunks; lane k issues the chunk's k-th copy.
    int n_issued = 0;
    long long cur_unit = -1;
    int grp = 0, item0 = 0, ob = 0;
    for (int i = 0; i < nr; ++i) {
      const uint32_t f = (uint32_t)tab[i].x;
      if (!(f & RD_CSTART)) continue;
      int cnt = 1;
      while (!((uint32_t)tab[i + cnt - 1].x & RD_CEND)) ++cnt;
      const long long unit = (unsigned)tab[i].y >> 9;
      const int rr = tab[i].y & 511;
      if (unit != cur_unit) {  // the tile changes with the unit only
        cur_unit = unit;
        const int jt = (int)(unit / P.m_tiles);
        ob = (int)(unit - (long long)jt * P.m_tiles);
        const int4 tl = P.tiles[jt];
        grp = tl.x;
        item0 = tl.y;
      }
      const int c = (int)rd_field(f, 8, 3);
      if (n_issued >= C::NC) {
        if (lane == 0) ok = mbar_wait_sleep(&c_empty[c], rd_field(f, 11, 1) ^ 1u, P.status);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
      }
      // this lane's copy: destination, source (bulk) or coordinates (TMA), bytes
      uint32_t bytes = 0;
      int kind = 0;  // 1 bulk, 2 TMA (bmap), 3 TMA (bmap_ext)
      void *dst = nullptr;
      const void *src = nullptr;
      int tx = 0;
      int k = lane;
      if (!(f & RD_EXT)) {
        const int kb_a = NP == 2 ? rr : 2 * rr;
        const int kb_b = NP == 2 ? rr + cnt : min(nkb, 2 * (rr + cnt));
        const int g_a = gidx[kb_a], g_b = gidx[kb_b - 1];
        if (k < NP) {
          kind = 1;
          bytes = (uint32_t)(kb_b - kb_a) * 4096;
          dst = ch_codes(c, k);
          src = reinterpret_cast<const uint8_t *>(P.codes[k]) + (((size_t)grp * P.m_tiles + ob) * nkb + kb_a) * 4096;
        } else if (k < 2 * NP) {
          const int p = k - NP;
          kind = 1;
          bytes = (uint32_t)(g_b - g_a + 1) * 512;
          dst = ch_sz(c, p);
          src = P.sz[p] + (((size_t)grp * P.m_tiles + ob) * (nkb * 128 / P.group) + g_a) * 128;
        } else {
          k -= 2 * NP;
          if (F8) {  // the two e4m3 pieces of each round's 128 K (one 128-byte box each)
            const int pos = k / 2, pc = k % 2;
            if (pos < cnt) {
              kind = 2;
              dst = ch_b(c, pos) + pc * C::ATOM;
              tx = pc * P.d_in + (rr + pos) * 128;
            }
          } else if (NP == 2) {  // fp16: two 64-wide atoms per round, shared by both projections
            const int pos = k / 2, a = k % 2;
            if (pos < cnt) {
              kind = 2;
              dst = ch_b(c, pos) + a * C::ATOM;
              tx = (rr + pos) * 128 + a * 64;
            }
          } else {  // one projection: two K blocks per round, two atoms each
            const int pos = k / 4, sl = (k / 2) % 2, a = k % 2;
            if (pos < cnt && 2 * (rr + pos) + sl < nkb) {
              kind = 2;
              dst = ch_b(c, pos) + (2 * sl + a) * C::ATOM;
              tx = (2 * (rr + pos) + sl) * 128 + a * 64;
            }
          }
          if (kind) bytes = C::ATOM;
        }
      } else {
        // extension rounds: the item rows' z (or a) columns of each valid slice
        constexpr int APS = C::EXT_W / 64;  // atoms per slice
        const int pos = k / (2 * APS), sl = (k / APS) % 2, a = k % APS;
        if (pos < cnt) {
          const uint32_t fp = (uint32_t)tab[i + pos].x;
          const int nat = ((int)rd_field(fp, sl ? 16 : 12, 4) + 3) / 4;
          if ((fp & (sl ? RD_V1 : RD_V0)) && a < nat) {
            const int p = NP == 2 ? sl : 0;
            kind = F8 ? 3 : 2;
            bytes = C::ATOM;
            dst = ch_b(c, pos) + (sl * APS + a) * C::ATOM;
            tx = P.ext_col[p] + (int)rd_field(fp, sl ? 30 : 28, 2) * C::EXT_W + a * 64;
          }
        }
      }
      const uint32_t total_bytes = __reduce_add_sync(0xffffffffu, bytes);
      if (lane == 0) mbar_arrive_expect_tx(&c_full[c], total_bytes);
      __syncwarp();
      if (kind == 1) {
        bulk_g2s(dst, src, bytes, &c_full[c]);
      } else if (kind == 2) {
        tc::tma_load_2d(dst, &P.bmap, tx, item0, &c_full[c]);
      } else if (kind == 3) {
        tc::tma_load_2d(dst, &P.bmap_ext, tx, item0, &c_full[c]);
      }
      ++n_issued;
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0)
      for (int j = n_issued > C::NC ? n_issued - C::NC : 0; j < n_issued; ++j)
        mbar_wait_sleep(&c_full[j % C::NC], (j / C::NC) & 1, P.status);
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc = tc::idesc_f16(BN);
    for (int i = 0; i < nr; ++i) {
      const uint32_t f = (uint32_t)tab[i].x;
      const int as = i % C::NA, ts = i % C::NT, c = (int)rd_field(f, 8, 3);
      const uint32_t acc_par = ((i / C::NT) - 1) & 1;
      const bool acc_ready = i < C::NT || mbar_test(&acc_free[ts], acc_par);
      if ((f & RD_CSTART) && !(ok = mbar_wait_sleep(&c_full[c], rd_field(f, 11, 1), P.status))) break;
      if (!(ok = mbar_wait_sleep(&a_full[as], (i / C::NA) & 1, P.status))) break;
      if (!acc_ready && !(ok = mbar_wait_sleep(&acc_free[ts], acc_par, P.status))) break;
      tc::fence_after();
      if (tc::elect_one()) {
        const uint64_t bd0 = tc::sdesc_sw128(smem_addr(ch_b(c, (int)rd_field(f, 6, 2))));
        const uint32_t a0 = tmem + as * C::A_COLS, d0 = tmem + C::ACC0 + ts * C::ACC_COLS;
        if (!(f & RD_EXT) && F8) {
          // e4m3: four K = 32 steps over 128 K per slice, both pieces of B into the same accumulator
#pragma unroll
          for (int sl = 0; sl < 2; ++sl)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
              for (int pc = 0; pc < 2; ++pc)
                tc::mma_ts_f8(d0 + sl * BN, a0 + sl * C::SCOLS + kk * 8, bd0 + (uint64_t)((pc * C::ATOM + kk * 32) >> 4),
                              idesc, (kk | pc) ? 1u : 0u);
        } else if (!(f & RD_EXT)) {
          // fp16: eight K = 16 steps per slice; the two projections of np = 2 share B atoms 0, 1
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            if (NP == 1 && sl == 1 && !(f & RD_V1)) break;
            const int atom0 = NP == 2 ? 0 : 2 * sl;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc::mma_ts(d0 + sl * BN, a0 + sl * C::SCOLS + kk * 8,
                         bd0 + (uint64_t)((((atom0 + kk / 4) * C::ATOM) + (kk % 4) * 32) >> 4), idesc, kk ? 1u : 0u);
          }
        } else {
          for (int sl = 0; sl < 2; ++sl) {
            if (!(f & (sl ? RD_V1 : RD_V0))) continue;
            const int nk = (int)rd_field(f, sl ? 16 : 12, 4);
            for (int kk = 0; kk < nk; ++kk)
              tc::mma_ts(d0 + sl * BN, a0 + sl * C::SCOLS + kk * 8,
                         bd0 + (uint64_t)((((sl * (C::EXT_W / 64) + kk / 4) * C::ATOM) + (kk % 4) * 32) >> 4), idesc,
                         kk ? 1u : 0u);
          }
        }
        // the operand slot is free once these MMAs have read it, the
        // accumulators are then ready to fold, and the chunk's activations are
        // done with after its last round
        tc::commit(&a_free[as]);
        tc::commit(&acc_full[ts]);
        if (f & RD_CEND) tc::commit(&c_empty[c]);
      }
      __syncwarp();
    }
    // all issued MMAs have retired before TMEM is released
    if (tc::elect_one()) tc::commit(drain);
    __syncwarp();
    mbar_wait_sleep(drain, 0, P.status);
  } else if (warp < 2 + DQ_DEC) {
    // ============================================================ decode
    // Two warps per TMEM lane quadrant (32 weight rows): warps 2..5 decode
    // slice 0 and warps 6..9 slice 1 of every round into its operand slot.
    // The slot's release is probed before the decode and awaited after it, so
    // the barrier's latency overlaps the decoding.
    const int dw = warp - 2;
    const int sl = dw / 4;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tc::lane_base(warp);
    // a round's stores complete while the warp decodes the next round: its
    // operand slot is then published (one round late)
    int prev_as = -1, prev_s = 0;
    auto arrive_prev = [&]() {
      if (prev_as < 0) return;
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[prev_as]);
        mbar_arrive(&s_full[prev_s]);
      }
      prev_as = -1;
    };
    for (int i = 0; i < nr && ok; ++i) {
      const int2 t = tab[i];
      const uint32_t f = (uint32_t)t.x;
      const int c = (int)rd_field(f, 8, 3);
      const int as = i % C::NA;
      const uint32_t free_par = ((i / C::NA) - 1) & 1;
      bool slot_free = i < C::NA || mbar_test(&a_free[as], free_par);
      if ((f & RD_CSTART) && !(ok = mbar_wait_sleep(&c_full[c], rd_field(f, 11, 1), P.status))) break;
      const uint32_t acol = tmem + lane_addr + as * C::A_COLS + sl * C::SCOLS;
      auto ensure_free = [&]() -> bool {
        arrive_prev();  // the previous round's stores landed while this round decoded
        if (!slot_free && !mbar_wait_sleep(&a_free[as], free_par, P.status)) return false;
        slot_free = true;
        tc::fence_after();
        return true;
      };
      if (f & (sl ? RD_V1 : RD_V0)) {
        if (!(f & RD_EXT)) {
          const int p = NP == 2 ? sl : 0;
          const uint8_t *cb = ch_codes(c, p) + rd_field(f, 20 + 2 * sl, 2) * 4096;
          const uint32_t szw = ch_sz(c, p)[rd_field(f, 24 + 2 * sl, 2) * 128 + row];
          // (the scale slot is written once the operand slot is free: the fold of
          // the slot's previous round is then done)
          auto put_scale = [&]() { sbuf[((i % C::NS) * 2 + sl) * 128 + row] = (unsigned short)(szw & 0xFFFFu); };
          uint2 wv[4];
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) wv[ks] = *reinterpret_cast<const uint2 *>(cb + ks * 1024 + row * 8);
          if constexpr (F8) {
            // e4m3 (q - z) through a 4-entry byte table per zero point: one PRMT per 4 weights.
            // The table for zero point z is bytes 3 - z .. 6 - z of e4m3(-3 .. 3); z comes out of
            // its fp16 bits by adding 1024 (ulp 1 there).
            const uint32_t zi = __half_as_ushort(__hadd(__ushort_as_half((unsigned short)(szw >> 16)),
                                                        __ushort_as_half((unsigned short)0x6400))) & 3u;
            const uint32_t tb = __byte_perm(0x00B8C0C4u, 0x00444038u, 0x6543u - zi * 0x1111u);
            uint32_t v[32];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // the four K slices of 32 (two words of 16 codes each)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint32_t w = h ? wv[ks].y : wv[ks].x;
                const uint32_t c0 = w & 0x33333333u, c1 = (w >> 2) & 0x33333333u;
                uint32_t *o = v + 8 * ks + 4 * h;
                o[0] = __byte_perm(tb, 0, c0);
                o[1] = __byte_perm(tb, 0, c0 >> 16);
                o[2] = __byte_perm(tb, 0, c1);
                o[3] = __byte_perm(tb, 0, c1 >> 16);
              }
            }
            if (!(ok = ensure_free())) break;
            put_scale();
            tc::st32(acol, v);
          } else {
            const __half2 z2 = __high2half2(u32_as_h2(szw));
            const __half2 nz[4] = {__hsub2(__float2half2_rn(-1024.f), z2), __hsub2(__float2half2_rn(-256.f), z2),
                                   __hsub2(__float2half2_rn(-64.f), z2), __hsub2(__float2half2_rn(-16.f), z2)};
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {  // K halves of 64: 32 TMEM columns each
              uint32_t v[32];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                dq_qz_word(wv[2 * hk + q].x, nz, v + 16 * q);
                dq_qz_word(wv[2 * hk + q].y, nz, v + 16 * q + 8);
              }
              if (hk == 0) {
                if (!(ok = ensure_free())) break;
                put_scale();
              }
              tc::st32(acol + hk * 32, v);
            }
            if (!ok) break;
          }
        } else {
          // rows of U_m: rank columns chunk * EXT_W ..
          const long long unit = (unsigned)t.y >> 9;
          const int jt = (int)(unit / P.m_tiles), ob = (int)(unit - (long long)jt * P.m_tiles);
          const int p = NP == 2 ? sl : 0;
          const int chunk = (int)rd_field(f, 28 + 2 * sl, 2);
          const __half *ur = P.u[p] + (((size_t)P.u_blk[p][P.tiles[jt].x] * P.m_tiles + ob) * 128 + row) * P.rank +
                             chunk * C::EXT_W;
          const int kmax = P.rank - chunk * C::EXT_W;
#pragma unroll
          for (int hk = 0; hk < C::EXT_W / 64; ++hk) {
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
            if (hk == 0 && !(ok = ensure_free())) break;
            tc::st32(acol + hk * 32, v);
          }
          if (!ok) break;
        }
      }
      // (a warp with nothing to write for the round still waits for the slot:
      // its arrival must not run ahead into the slot's previous phase)
      if (!(ok = ensure_free())) break;
      // the round's arrival waits for its stores, after the next round's decode
      prev_as = as;
      prev_s = i % C::NS;
      // the chunk's codes are decoded: the producer may refill its slot
      if ((f & RD_CEND) && lane == 0) mbar_arrive(&c_empty[c]);
    }
    if (ok) arrive_prev();
  } else {
    // ============================================================ fold + epilogue
    // One warp per TMEM lane quadrant (32 weight rows): it folds both slices'
    // accumulators of every round into registers with the group scale, so a
    // unit's two slices meet in the same thread, and stores the unit's result.
    const int fw = warp - 2 - DQ_DEC;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tc::lane_base(warp);
    float acc0[BN], acc1[BN];  // np = 2: gate, up; np = 1: the two slices' partial sums
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      acc0[c] = 0.f;
      acc1[c] = 0.f;
    }

    // ---- end of a unit's rounds in this CTA: store the result (whole unit) or
    // a piece (unit cut between CTAs; the CTA finishing last sums them)
    auto unit_end = [&](const int unit, const int jt, const int ob) -> void {
      const long long ustart = (long long)unit * R, uend = ustart + R;
      const bool whole = ustart >= r0 && uend <= r1;
      const int4 t = P.tiles[jt];
      const int item0 = t.y, nitems = t.z;
      const int o = ob * 128 + row;
      // per-item factors, one per lane (items < 32), handed out by shuffles
      const float xs_l = (F8 && lane < nitems) ? __ldg(P.xs + item0 + lane) : 1.f;
      const float rs_l = (NP == 2 && P.row_scale && lane < nitems) ? __ldg(P.row_scale + item0 + lane) : 1.f;
      // the final result of item column n: np = 2: silu(gate) * up * row scale (fp16) or both in
      // fp32; np = 1: the sum of both slices (fp32).  Called by the whole warp with the same n.
      auto store = [&](int n, float g, float u) {
        const float xs = __shfl_sync(0xffffffffu, xs_l, n), rs = __shfl_sync(0xffffffffu, rs_l, n);
        if (n >= nitems || o >= P.d_out) return;
        if (F8) {  // the activations were scaled by 2^e per item
          g *= xs;
          u *= xs;
        }
        if (NP == 2 && P.epi == EPI_STORE2_F32) {
          reinterpret_cast<float *>(P.out)[(size_t)(item0 + n) * P.ldo + o] = g;
          reinterpret_cast<float *>(P.out2)[(size_t)(item0 + n) * P.ldo + o] = u;
        } else if (NP == 2) {
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
        named_sync(1, DQ_FW * 32);
        const int c_first = cta_of(ustart, total, gridDim.x), c_last = cta_of(uend - 1, total, gridDim.x);
        // CTAs with an empty range (fewer rounds than CTAs) leave no piece
        int pieces = 0;
        for (int cc = c_first; cc <= c_last; ++cc)
          pieces += range_begin(total, cc + 1, gridDim.x) > range_begin(total, cc, gridDim.x);
        if (fw == 0 && lane == 0) *flag = atomicAdd(&P.counters[unit], 1) == pieces - 1;
        named_sync(1, DQ_FW * 32);
        fin = *flag != 0;
        if (fin) {
          // the last piece in: sum all pieces of the unit in CTA order (the
          // range arithmetic once per piece, not per column)
          __threadfence();
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            acc0[c] = 0.f;
            acc1[c] = 0.f;
          }
          for (int cc = c_first; cc <= c_last; ++cc) {
            const long long b = range_begin(total, cc, gridDim.x);
            if (range_begin(total, cc + 1, gridDim.x) == b) continue;
            const int s2 = (b / R == unit) ? 0 : 1;  // the unit is cta cc's first (slot 0) or last
            const float *q = P.part + ((size_t)cc * 2 + s2) * NP * BN * 128;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
              acc0[c] += __ldcg(q + c * 128 + row);
              if (NP == 2) acc1[c] += __ldcg(q + (BN + c) * 128 + row);
            }
          }
#pragma unroll
          for (int c = 0; c < BN; ++c) store(c, acc0[c], acc1[c]);
          if (fw == 0 && lane == 0) P.counters[unit] = 0;
        }
      }
      // weighted top-k combine: the slot weights are inside h, so the layer
      // output of a token is the plain sum of its slots' rows
      if (NP == 1 && P.combine && fin) {
        __threadfence();
        named_sync(1, DQ_FW * 32);
        const int tid = ((warp & 3) * 32) + lane;  // 0 .. 127
        if (tid < nitems) {
          const int tok = __ldg(P.slot_tok + item0 + tid);
          fin_tok[tid] = atomicAdd(&P.tok_counters[tok * P.m_tiles + ob], 1) == P.top_k - 1;
        }
        named_sync(1, DQ_FW * 32);
        __threadfence();
        const float *yb = reinterpret_cast<const float *>(P.out);
        for (int n = 0; n < nitems; ++n) {
          if (!fin_tok[n]) continue;
          const int tok = __ldg(P.slot_tok + item0 + n);
          const int oo = ob * 128 + tid;
          if (oo >= P.d_out) continue;
          float y = P.yshared ? __ldg(P.yshared + (size_t)tok * P.ldo + oo) : 0.f;
          for (int j = 0; j < P.top_k; ++j)
            y += __ldcg(yb + (size_t)__ldg(P.slot_of_pair + tok * P.top_k + j) * P.ldo + oo);
          P.out_tok[(size_t)tok * P.ldo + oo] = __float2bfloat16_rn(y);
        }
        named_sync(1, DQ_FW * 32);  // fin_tok is reused by the next unit
      }
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        acc0[c] = 0.f;
        acc1[c] = 0.f;
      }
    };

    // fold one slice's accumulator (BN columns at TMEM column base) into acc
    auto fold = [&](uint32_t base, float s, float (&acc)[BN]) {
      uint32_t d[BN];
      if constexpr (BN == 32) {
        tc::ld32_nowait(base, d);
      } else {
        tc::ld16_nowait(base, d);
      }
      tc::wait_ld();
#pragma unroll
      for (int c = 0; c < BN; ++c) acc[c] = fmaf(__uint_as_float(d[c]), s, acc[c]);
    };

    for (int i = 0; i < nr && ok; ++i) {
      const int ts = i % C::NT;
      const int2 t = tab[i];
      const uint32_t f = (uint32_t)t.x;
      const int c = (int)rd_field(f, 8, 3);
      // this row's scale of each slice (1 for the U_m extension), handed over by the decode warps
      const uint32_t s_par = (i / C::NS) & 1;
      const bool s_ready = mbar_test(&s_full[i % C::NS], s_par);
      if (!(ok = mbar_wait_sleep(&acc_full[ts], (i / C::NT) & 1, P.status))) break;
      if (!s_ready && !(ok = mbar_wait_sleep(&s_full[i % C::NS], s_par, P.status))) break;
      tc::fence_after();
      float s0 = 1.f, s1 = 1.f;
      if (!(f & RD_EXT)) {
        s0 = __half2float(__ushort_as_half(sbuf[((i % C::NS) * 2 + 0) * 128 + row]));
        s1 = __half2float(__ushort_as_half(sbuf[((i % C::NS) * 2 + 1) * 128 + row]));
      }
      // tcgen05.ld is warp-collective: the decision is the warp's (the slice
      // was valid in round i), never a lane's (padding rows have scale 0)
      const uint32_t base = tmem + lane_addr + C::ACC0 + ts * C::ACC_COLS;
      if (f & RD_V0) fold(base, s0, acc0);
      if (f & RD_V1) fold(base + BN, s1, acc1);
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[ts]);
      if (f & RD_UEND) {
        const long long unit = (unsigned)t.y >> 9;
        const int jt = (int)(unit / P.m_tiles);
        unit_end((int)unit, jt, (int)(unit - (long long)jt * P.m_tiles));
      }
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

template <int NP, int BN, bool F8 = false>
cudaError_t launch_dq(const DqArgs &a, cudaStream_t stream) {
  using C = DqCfg<NP, BN, F8>;
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

bool dq_fits(int max_tiles, int m_tiles, int d_in, int rank) {
  // the most rounds a unit can have (two-projection launches: one K block per round)
  const long long R = d_in / 128 + (rank + 127) / 128;
  const long long total = (long long)max_tiles * m_tiles * R;
  return (total + DQ_GRID - 1) / DQ_GRID <= DQ_MAX_ROUNDS;
}

cudaError_t launch_gemm_dq(const DqArgs &a, int np, int bn, cudaStream_t stream) {
  if (a.m_tiles <= 0 || a.group % 128 != 0 || a.d_in % 128 != 0 || a.d_in > 128 * 256 || a.rank < 0 || a.rank > 256 ||
      !dq_fits(a.max_tiles, a.m_tiles, a.d_in, a.rank))
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
