// Repacking of the stored TileQ format into the layouts the GEMM reads.
// Rows are grouped in blocks of 128 (eight m16 tiles, one per consumer warp),
// so that one pipeline stage of a CTA is one contiguous bulk copy.
#include "kernels.cuh"

namespace tileq {

// 2-bit codes [K][d_out][d_in/16] (element j at bits 2*(j%16)) ->
// [K][R/128][d_in/128][8 warps][32 lanes] uint4.  Word w of a lane covers k32
// block w of the k128 block; within it, k16 step s and fragment register i keep
// the (lo, hi) codes at bits (8s + 2i, 16 + 8s + 2i).  Register i is the
// m16n8k16 A-fragment register: rows r0 = l/4 (+8 for odd i), columns
// 2*(l%4) (+8 for i >= 2).  Rows past d_out hold code 0.
__global__ void pack_codes_kernel(const uint32_t *codes, uint4 *out, int K, int d_out, int d_in) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nkb = d_in / 128, n128 = pad128(d_out) / 128, wpr = d_in / 16;
  const long long total = (long long)K * n128 * nkb * 8 * 32;
  if (gid >= total) return;
  const int lane = (int)(gid % 32);
  long long rest = gid / 32;
  const int w8 = (int)(rest % 8);
  rest /= 8;
  const int kb = (int)(rest % nkb);
  rest /= nkb;
  const int ob = (int)(rest % n128);
  const int e = (int)(rest / n128);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  auto code = [&](int row, int col) -> uint32_t {
    if (row >= d_out) return 0u;
    const uint32_t word = codes[((size_t)e * d_out + row) * wpr + col / 16];
    return (word >> (2 * (col % 16))) & 3u;
  };
  uint32_t words[4];
  for (int w = 0; w < 4; ++w) {
    uint32_t acc = 0;
    for (int s = 0; s < 2; ++s) {
      const int ks = kb * 128 + w * 32 + s * 16;
      for (int i = 0; i < 4; ++i) {
        const int row = ob * 128 + w8 * 16 + r0 + 8 * (i & 1);
        const int col = ks + c + 8 * (i >> 1);
        acc |= code(row, col) << (8 * s + 2 * i);
        acc |= code(row, col + 1) << (16 + 8 * s + 2 * i);
      }
    }
    words[w] = acc;
  }
  out[gid] = make_uint4(words[0], words[1], words[2], words[3]);
}

// 3-bit codes' high bits [K][d_out][d_in/32] (element j at bit j%32) ->
// [K][R/128][d_in/128][8 warps][32 lanes] uint2, beside pack_codes_kernel's
// layout: word p of a lane holds the high bits of its code words 2p and 2p+1.
// For code word 2p, k16 step s and fragment register i, the (lo, hi) codes'
// bits sit at (2 + 2i + s, 18 + 2i + s): after the decoder's shift by s, bit
// 2i+2 lies just above the 2-bit field of register i.  Code word 2p+1 uses the
// same positions rotated left by 8 (the 32 positions are all distinct).
__global__ void pack_codes_hi_kernel(const uint32_t *hi, uint2 *out, int K, int d_out, int d_in) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nkb = d_in / 128, n128 = pad128(d_out) / 128, wpr = d_in / 32;
  const long long total = (long long)K * n128 * nkb * 8 * 32;
  if (gid >= total) return;
  const int lane = (int)(gid % 32);
  long long rest = gid / 32;
  const int w8 = (int)(rest % 8);
  rest /= 8;
  const int kb = (int)(rest % nkb);
  rest /= nkb;
  const int ob = (int)(rest % n128);
  const int e = (int)(rest / n128);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  auto bit = [&](int row, int col) -> uint32_t {
    if (row >= d_out) return 0u;
    return (hi[((size_t)e * d_out + row) * wpr + col / 32] >> (col % 32)) & 1u;
  };
  uint32_t words[2] = {0u, 0u};
  for (int w = 0; w < 4; ++w) {
    uint32_t acc = 0;
    for (int s = 0; s < 2; ++s) {
      const int ks = kb * 128 + w * 32 + s * 16;
      for (int i = 0; i < 4; ++i) {
        const int row = ob * 128 + w8 * 16 + r0 + 8 * (i & 1);
        const int col = ks + c + 8 * (i >> 1);
        acc |= bit(row, col) << (2 + 2 * i + s);
        acc |= bit(row, col + 1) << (18 + 2 * i + s);
      }
    }
    if (w & 1) acc = (acc << 8) | (acc >> 24);
    words[w >> 1] |= acc;
  }
  out[gid] = make_uint2(words[0], words[1]);
}

// scales fp16 [K][d_out][G], zeros [K][d_out][ceil(G/4)] (2-bit; 3-bit:
// [K][d_out][ceil(G/2)], 4-bit fields) ->
// [K][R/128][G][8 warps][16 rows] u32 = {low half: scale bits, high half: fp16(z)};
// rows past d_out hold scale 0.
__global__ void pack_sz_kernel(const __half *scales, const uint8_t *zeros, uint32_t *out, int K,
                               int d_out, int G, int bits) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int n128 = pad128(d_out) / 128;
  const long long total = (long long)K * n128 * G * 128;
  if (gid >= total) return;
  const int r = (int)(gid % 16);
  long long rest = gid / 16;
  const int w8 = (int)(rest % 8);
  rest /= 8;
  const int grp = (int)(rest % G);
  rest /= G;
  const int ob = (int)(rest % n128);
  const int e = (int)(rest / n128);
  const int row = ob * 128 + w8 * 16 + r;
  if (row >= d_out) {
    out[gid] = 0u;
    return;
  }
  const __half s = scales[((size_t)e * d_out + row) * G + grp];
  uint32_t z;
  if (bits == 3) {
    const int zb = (G + 1) / 2;
    z = (zeros[((size_t)e * d_out + row) * zb + grp / 2] >> (4 * (grp % 2))) & 7u;
  } else {
    const int zb = (G + 3) / 4;
    z = (zeros[((size_t)e * d_out + row) * zb + grp / 4] >> (2 * (grp % 4))) & 3u;
  }
  const __half zh = __uint2half_rn(z);
  const uint32_t lo = *reinterpret_cast<const uint16_t *>(&s);
  const uint32_t hi = *reinterpret_cast<const uint16_t *>(&zh);
  out[gid] = lo | (hi << 16);
}

// bf16 matrix blocks S_b[R][C] -> fp16 A fragments
// [nblk][R/128][C/(16*kb)][8 warps][kb k16 steps][32 lanes] uint4 (zero padded).
__global__ void pack_frag_kernel(const __nv_bfloat16 *src, long long bs, long long rs, long long cs,
                                 int nblk, int R, int C, int kb, uint4 *out) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int n128 = pad128(R) / 128;
  const int nkb = (C + 16 * kb - 1) / (16 * kb);
  const long long total = (long long)nblk * n128 * nkb * 8 * kb * 32;
  if (gid >= total) return;
  const int lane = (int)(gid % 32);
  long long rest = gid / 32;
  const int ks = (int)(rest % kb);
  rest /= kb;
  const int w8 = (int)(rest % 8);
  rest /= 8;
  const int kbi = (int)(rest % nkb);
  rest /= nkb;
  const int ob = (int)(rest % n128);
  const int b = (int)(rest / n128);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  const __nv_bfloat16 *base = src + b * bs;
  auto at = [&](int row, int col) -> float {
    if (row >= R || col >= C) return 0.f;
    return __bfloat162float(base[row * rs + col * cs]);
  };
  uint32_t regs[4];
  for (int i = 0; i < 4; ++i) {
    const int row = ob * 128 + w8 * 16 + r0 + 8 * (i & 1);
    const int col = (kbi * kb + ks) * 16 + c + 8 * (i >> 1);
    const __half2 h = __floats2half2_rn(at(row, col), at(row, col + 1));
    regs[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  out[gid] = make_uint4(regs[0], regs[1], regs[2], regs[3]);
}

__global__ void pack_codes_tc_kernel(const uint32_t *codes, uint32_t *out, int K, int d_out, int d_in) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nkb = d_in / 128, n128 = pad128(d_out) / 128, wpr = d_in / 16;
  const long long total = (long long)K * n128 * nkb * 128 * 8;
  if (gid >= total) return;
  // word index within the 4 KB block of (expert, row block, k block):
  // (part * 128 + row) * 2 + wi, part = 32-element K slice, wi = 16-element half
  const int wi = (int)(gid % 2);
  const int r = (int)((gid / 2) % 128);
  const int part = (int)((gid / 256) % 4);
  const int w = part * 2 + wi;
  long long rest = gid / 1024;
  const int kb = (int)(rest % nkb);
  rest /= nkb;
  const int ob = (int)(rest % n128);
  const int e = (int)(rest / n128);
  const int row = ob * 128 + r;
  uint32_t acc = 0;
  if (row < d_out) {
    for (int p = 0; p < 8; ++p)
      for (int h = 0; h < 2; ++h) {
        const int col = kb * 128 + w * 16 + 2 * p + h;
        const uint32_t word = codes[((size_t)e * d_out + row) * wpr + col / 16];
        const uint32_t q = (word >> (2 * (col % 16))) & 3u;
        acc |= q << ((h ? 16 : 0) + 2 * (p % 4) + 8 * (p / 4));
      }
  }
  out[gid] = acc;
}

// 3-bit codes' high bits [K][d_out][d_in/32] -> [K][R/128][d_in/128][4 slices][128 rows]
// u32, beside pack_codes_tc_kernel's layout: the word of (slice, row) holds
// the high bits of its two code words (16-element halves wi = 0, 1).  Pair p,
// half h of code word 0 at bit (h ? 16 : 0) + 2 + 2*(p%4) + p/4, just above the
// 2-bit field once the decoder has shifted by p/4; code word 1's bits rotated
// left by 8.
__global__ void pack_codes_tc_hi_kernel(const uint32_t *hi, uint32_t *out, int K, int d_out, int d_in) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nkb = d_in / 128, n128 = pad128(d_out) / 128, wpr = d_in / 32;
  const long long total = (long long)K * n128 * nkb * 4 * 128;
  if (gid >= total) return;
  const int r = (int)(gid % 128);
  const int part = (int)((gid / 128) % 4);
  long long rest = gid / 512;
  const int kb = (int)(rest % nkb);
  rest /= nkb;
  const int ob = (int)(rest % n128);
  const int e = (int)(rest / n128);
  const int row = ob * 128 + r;
  uint32_t acc = 0;
  if (row < d_out) {
    for (int wi = 0; wi < 2; ++wi) {
      uint32_t a = 0;
      for (int p = 0; p < 8; ++p)
        for (int h = 0; h < 2; ++h) {
          const int col = kb * 128 + (part * 2 + wi) * 16 + 2 * p + h;
          const uint32_t b = (hi[((size_t)e * d_out + row) * wpr + col / 32] >> (col % 32)) & 1u;
          a |= b << ((h ? 16 : 0) + 2 + 2 * (p % 4) + p / 4);
        }
      if (wi) a = (a << 8) | (a >> 24);
      acc |= a;
    }
  }
  out[gid] = acc;
}

// Sigma [r] -> [n][rp] (rp = r rounded up to 128; zeros past r): the column
// scales of the projection onto all n grid columns at once.
__global__ void expand_sigma_kernel(const float *sigma, int r, int rp, int n, float *out) {
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n * rp) return;
  const int i = gid % rp;
  out[gid] = i < r ? sigma[i] : 0.f;
}

__global__ void pack_rows_f16_kernel(const __nv_bfloat16 *src, int nblk, int R, int C, __half *out) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int Rp = pad128(R);
  const long long total = (long long)nblk * Rp * C;
  if (gid >= total) return;
  const int c = (int)(gid % C);
  long long rest = gid / C;
  const int r = (int)(rest % Rp);
  const int b = (int)(rest / Rp);
  out[gid] = r < R ? __float2half_rn(__bfloat162float(src[((size_t)b * R + r) * C + c])) : __float2half_rn(0.f);
}

// V [N][d_in][r] (bf16) -> V_n^T rows in fp16, [N][pad128(r)][d_in] (zero rows
// past r): the row-major A operand of the tensor-core product z = V_n^T x.
__global__ void pack_vt_rows_kernel(const __nv_bfloat16 *V, int N, int r, int d_in, __half *out) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int rp = pad128(r);
  const long long total = (long long)N * rp * d_in;
  if (gid >= total) return;
  const int k = (int)(gid % d_in);
  long long rest = gid / d_in;
  const int i = (int)(rest % rp);
  const int n = (int)(rest / rp);
  out[gid] = i < r ? __float2half_rn(__bfloat162float(V[((size_t)n * d_in + k) * r + i])) : __float2half_rn(0.f);
}

}  // namespace tileq
