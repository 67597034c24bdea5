// Repacking of the stored TileQ format into the layouts the GEMM reads.
#include "kernels.cuh"

namespace tileq {

// 2-bit codes [K][d_out][d_in/16] (element j at bits 2*(j%16)) ->
// [K][d_out/16][d_in/128][32 lanes] uint4.  Word w of lane l covers k32 block w
// of the k128 block; within it, k16 step s and fragment register i keep the
// (lo, hi) codes at bits (8s + 2i, 16 + 8s + 2i).  Register i is the m16n8k16
// A-fragment register: rows r0 = l/4 (+8 for odd i), columns 2*(l%4) (+8 for i >= 2).
__global__ void pack_codes_kernel(const uint32_t *codes, uint4 *out, int K, int d_out, int d_in) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nkb = d_in / 128, n16 = d_out / 16, wpr = d_in / 16;
  const long long total = (long long)K * n16 * nkb * 32;
  if (gid >= total) return;
  const int lane = (int)(gid % 32);
  long long rest = gid / 32;
  const int kb = (int)(rest % nkb);
  rest /= nkb;
  const int o16 = (int)(rest % n16);
  const int e = (int)(rest / n16);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  auto code = [&](int row, int col) -> uint32_t {
    const uint32_t word = codes[((size_t)e * d_out + row) * wpr + col / 16];
    return (word >> (2 * (col % 16))) & 3u;
  };
  uint32_t words[4];
  for (int w = 0; w < 4; ++w) {
    uint32_t acc = 0;
    for (int s = 0; s < 2; ++s) {
      const int ks = kb * 128 + w * 32 + s * 16;
      for (int i = 0; i < 4; ++i) {
        const int row = o16 * 16 + r0 + 8 * (i & 1);
        const int col = ks + c + 8 * (i >> 1);
        acc |= code(row, col) << (8 * s + 2 * i);
        acc |= code(row, col + 1) << (16 + 8 * s + 2 * i);
      }
    }
    words[w] = acc;
  }
  out[gid] = make_uint4(words[0], words[1], words[2], words[3]);
}

// scales fp16 [K][d_out][G], zeros [K][d_out][ceil(G/4)] ->
// [K][d_out/16][G][16 rows] u32 = {low half: scale bits, high half: fp16(z)}.
__global__ void pack_sz_kernel(const __half *scales, const uint8_t *zeros, uint32_t *out, int K,
                               int d_out, int G) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)K * d_out * G;
  if (gid >= total) return;
  const int r = (int)(gid % 16);
  long long rest = gid / 16;
  const int grp = (int)(rest % G);
  rest /= G;
  const int o16 = (int)(rest % (d_out / 16));
  const int e = (int)(rest / (d_out / 16));
  const int row = o16 * 16 + r;
  const int zb = (G + 3) / 4;
  const __half s = scales[((size_t)e * d_out + row) * G + grp];
  const uint32_t z = (zeros[((size_t)e * d_out + row) * zb + grp / 4] >> (2 * (grp % 4))) & 3u;
  const __half zh = __uint2half_rn(z);
  const uint32_t lo = *reinterpret_cast<const uint16_t *>(&s);
  const uint32_t hi = *reinterpret_cast<const uint16_t *>(&zh);
  out[gid] = lo | (hi << 16);
}

__global__ void pack_frag_kernel(const __nv_bfloat16 *src, long long bs, long long rs, long long cs,
                                 int nblk, int R, int C, uint4 *out) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int r16 = R / 16, c16 = C / 16;
  const long long total = (long long)nblk * r16 * c16 * 32;
  if (gid >= total) return;
  const int lane = (int)(gid % 32);
  long long rest = gid / 32;
  const int tj = (int)(rest % c16);
  rest /= c16;
  const int ti = (int)(rest % r16);
  const int b = (int)(rest / r16);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  const __nv_bfloat16 *base = src + b * bs;
  uint32_t regs[4];
  for (int i = 0; i < 4; ++i) {
    const int row = ti * 16 + r0 + 8 * (i & 1);
    const int col = tj * 16 + c + 8 * (i >> 1);
    const float lo = __bfloat162float(base[row * rs + col * cs]);
    const float hi = __bfloat162float(base[row * rs + (col + 1) * cs]);
    const __half2 h = __floats2half2_rn(lo, hi);
    regs[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  out[gid] = make_uint4(regs[0], regs[1], regs[2], regs[3]);
}

}  // namespace tileq
