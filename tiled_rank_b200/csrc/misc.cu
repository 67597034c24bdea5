// Small element-wise kernels of the TileQ forward: the in-place accumulation
// of the low-rank projections per (token, grid row), the weighted top-k
// combine / unpermute, and the helpers of the unfused comparison path.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace tileq {

// For the designated slot s of each (token t, grid row m):
//   out[s][col + i] = sum over the token's slots j whose expert sits in row m of
//       w_j * zcol[zidx(slot(t,j))][i]     (linear layer: z per (token, column))
//   or  zslot[slot(t,j)][i]                (per-slot rows with the weight already
//                                           applied; the forward does not use this
//                                           source: its SwiGLU down projection adds
//                                           U_m z' per slot in the K extension),
// and zeros for every other slot.  TileQ paper, section 2.2: routing weights
// select the active tiles of the projected [T, N, r] tensor and an in-place
// buffer accumulates them per grid row, so that the shared left factor U_m is
// applied once per (token, row); here the buffer lives in the K-extension
// columns of the next GEMM's activation matrix.
// One warp per slot.  The token's k pairs are looked up once (lane j holds
// pair j's slot, weight and z row, or -1 outside grid row m) and broadcast;
// each lane then sums four consecutive elements over the pairs, all pairs'
// loads in flight, in pair order and split order.
__global__ void __launch_bounds__(256) lr_accumulate_kernel(LrAccArgs a) {
  pdl_wait_and_release();
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.P) return;
  const int s = (int)gw;
  const int r4 = a.r / 4;
  __half2 *dst = reinterpret_cast<__half2 *>(a.out + (size_t)s * a.ld + a.col);
  if (a.aidx[s] < 0) {
    for (int c = lane; c < r4; c += 32) {
      dst[2 * c] = __floats2half2_rn(0.f, 0.f);
      dst[2 * c + 1] = __floats2half2_rn(0.f, 0.f);
    }
    return;
  }
  const int p0 = a.sorted_pairs[s];
  const int t = p0 / a.k;
  const int m = a.m_of[a.topk_idx[p0]];
  int my_slot = -1, my_row = 0;
  float my_w = 0.f;
  if (lane < a.k) {
    const int p = t * a.k + lane;
    if (a.m_of[a.topk_idx[p]] == m) {
      my_slot = a.slot_of_pair[p];
      my_w = a.topk_w[p];
      my_row = a.zslot ? my_slot : a.zidx[my_slot];
    }
  }
  int slot[kMaxTopK], zrow[kMaxTopK];
  float w[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    slot[j] = __shfl_sync(0xffffffffu, my_slot, j);
    zrow[j] = __shfl_sync(0xffffffffu, my_row, j);
    w[j] = __shfl_sync(0xffffffffu, my_w, j);
  }
  const float *zbase = a.zslot ? a.zslot : a.zcol;
  const size_t zstride = a.zslot ? (size_t)a.r : (size_t)a.zld;
  for (int c = lane; c < r4; c += 32) {
    float4 z[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      z[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < a.k && slot[j] >= 0) {
        const float *zp = zbase + (size_t)zrow[j] * zstride + 4 * c;
        for (int sp = 0; sp < a.zks; ++sp) {  // K-split partials in split order
          const float4 q = *reinterpret_cast<const float4 *>(zp + (size_t)sp * a.zsplit);
          z[j].x += q.x; z[j].y += q.y; z[j].z += q.z; z[j].w += q.w;
        }
      }
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k && slot[j] >= 0) {
        const float f = a.zslot ? 1.f : w[j];
        acc.x += f * z[j].x; acc.y += f * z[j].y; acc.z += f * z[j].z; acc.w += f * z[j].w;
      }
    }
    dst[2 * c] = half2_checked(acc.x, acc.y, a.status);
    dst[2 * c + 1] = half2_checked(acc.z, acc.w, a.status);
  }
}

// x_ext[s] = [x16[tok(s)] | z0[zidx0[s]] | z1[zidx1[s]]]  (fp16, 8-element chunks)
// Eight z values of row s: the sum of the K-split partials in split order, to fp16.
__device__ __forceinline__ uint4 z_chunk(const GatherExtArgs &a, int s, int zc) {
  const int p = zc / (a.r / 8), cc = zc % (a.r / 8);
  const float *z = a.z[p] + (size_t)a.zidx[p][s] * a.zld + cc * 8;
  float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
  for (int sp0 = 0; sp0 < a.zks; sp0 += 8) {
    // eight splits' loads in flight, then summed in split order
    float4 l[8], h[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool in = sp0 + u < a.zks;
      const float4 *q = reinterpret_cast<const float4 *>(z + (size_t)(sp0 + u) * a.zsplit);
      l[u] = in ? q[0] : make_float4(0.f, 0.f, 0.f, 0.f);
      h[u] = in ? q[1] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      lo.x += l[u].x; lo.y += l[u].y; lo.z += l[u].z; lo.w += l[u].w;
      hi.x += h[u].x; hi.y += h[u].y; hi.z += h[u].z; hi.w += h[u].w;
    }
  }
  uint4 v;
  __half2 *o = reinterpret_cast<__half2 *>(&v);
  o[0] = half2_checked(lo.x, lo.y, a.status);
  o[1] = half2_checked(lo.z, lo.w, a.status);
  o[2] = half2_checked(hi.x, hi.y, a.status);
  o[3] = half2_checked(hi.z, hi.w, a.status);
  return v;
}

// Grid-stride over T * (d/8) token-major x chunks (each read once and written
// to the token's k slot rows), then P * (nz*r/8) slot-major z chunks;
// kGatherUnroll items per thread in flight.
__global__ void __launch_bounds__(256) gather_ext_kernel(GatherExtArgs a) {
  pdl_wait_and_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long G = (long long)gridDim.x * blockDim.x;
  const int nz = a.z[0] ? (a.z[1] ? 2 : 1) : 0;
  const int xc = a.d / 8, zcn = nz * (a.r / 8);
  const long long nx = (long long)a.T * xc;
  const long long total = nx + (long long)a.P * zcn;
  for (long long c0 = gid; c0 < total; c0 += kGatherUnroll * G) {
    uint4 v[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const long long i = c0 + u * G;
      if (i < nx) {
        const int t = (int)(i / xc), c = (int)(i % xc);
        v[u] = __ldg(reinterpret_cast<const uint4 *>(a.x16 + (size_t)t * a.d) + c);
      } else if (i < total) {
        const long long iz = i - nx;
        v[u] = z_chunk(a, (int)(iz / zcn), (int)(iz % zcn));
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const long long i = c0 + u * G;
      if (i < nx) {
        const int t = (int)(i / xc), c = (int)(i % xc);
        for (int j = 0; j < a.k; ++j) {
          const int s = a.slot_of_pair[t * a.k + j];
          reinterpret_cast<uint4 *>(a.out + (size_t)s * a.ld)[c] = v[u];
        }
      } else if (i < total) {
        const long long iz = i - nx;
        const int s = (int)(iz / zcn), c = xc + (int)(iz % zcn);
        reinterpret_cast<uint4 *>(a.out + (size_t)s * a.ld)[c] = v[u];
      }
    }
  }
}

// e4m3 pieces of one 16-element block of a scaled activation row: p0 + p1.
__device__ __forceinline__ void e4m3_pieces(const float (&v)[16], uint4 &p0, uint4 &p1) {
  uint32_t w0[4], w1[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // stored position 4j + b holds element j + 4b (the order of the decoded weights)
    float f0[4], f1[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float x = v[j + 4 * b];
      const __nv_fp8_storage_t h = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
      const float hx = __half2float(__half(__nv_cvt_fp8_to_halfraw(h, __NV_E4M3)));
      f0[b] = hx;
      f1[b] = x - hx;
    }
    const __nv_fp8x2_storage_t a01 = __nv_cvt_float2_to_fp8x2(make_float2(f0[0], f0[1]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t a23 = __nv_cvt_float2_to_fp8x2(make_float2(f0[2], f0[3]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t b01 = __nv_cvt_float2_to_fp8x2(make_float2(f1[0], f1[1]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t b23 = __nv_cvt_float2_to_fp8x2(make_float2(f1[2], f1[3]), __NV_SATFINITE, __NV_E4M3);
    w0[j] = (uint32_t)a01 | ((uint32_t)a23 << 16);
    w1[j] = (uint32_t)b01 | ((uint32_t)b23 << 16);
  }
  p0 = make_uint4(w0[0], w0[1], w0[2], w0[3]);
  p1 = make_uint4(w1[0], w1[1], w1[2], w1[3]);
}

__global__ void __launch_bounds__(256) gather_x8_kernel(GatherX8Args a) {
  pdl_wait_and_release();
  __shared__ float red[8];
  const int t = blockIdx.x;
  if (t >= a.T) return;
  const __half *xr = a.x16 + (size_t)t * a.d;
  const int nb = a.d / 16;
  // the row maximum of |x|
  float m = 0.f;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    const uint4 *q = reinterpret_cast<const uint4 *>(xr + b * 16);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = __ldg(q + h);
      const __half2 *hh = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(hh[i]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  int ex = 0;
  if (m > 0.f) frexpf(m, &ex);            // m = f * 2^ex, f in [0.5, 1)
  const int e = m > 0.f ? 8 - ex : 0;     // m * 2^e in [128, 256)
  const float up = ldexpf(1.f, e), down = ldexpf(1.f, -e);
  int slots[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) slots[j] = j < a.k ? __ldg(a.slot_of_pair + t * a.k + j) : 0;
  if (threadIdx.x < a.k) a.xs[slots[threadIdx.x]] = down;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    float v[16];
    const uint4 *q = reinterpret_cast<const uint4 *>(xr + b * 16);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = __ldg(q + h);
      const __half2 *hh = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(hh[i]);
        v[8 * h + 2 * i] = f.x * up;
        v[8 * h + 2 * i + 1] = f.y * up;
      }
    }
    uint4 p0, p1;
    e4m3_pieces(v, p0, p1);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j >= a.k) break;
      uint8_t *row = a.x8 + (size_t)slots[j] * 2 * a.d;
      reinterpret_cast<uint4 *>(row)[b] = p0;
      reinterpret_cast<uint4 *>(row + a.d)[b] = p1;
    }
  }
  // z rows of the token's slots, scaled like x, into the extension columns
  const int nz = a.z[0] ? (a.z[1] ? 2 : 1) : 0;
  const int per = nz * a.r;
  for (int idx = threadIdx.x; idx < a.k * per; idx += blockDim.x) {
    const int j = idx / per, c = idx % per, p = c / a.r, i = c % a.r;
    const int s = slots[j];
    const float *zp = a.z[p] + (size_t)a.zidx[p][s] * a.zld + i;
    float acc = 0.f;
    for (int sp = 0; sp < a.zks; ++sp) acc += zp[(size_t)sp * a.zsplit];
    a.xext[(size_t)s * a.ld + a.d + c] = half_checked(acc * up, a.status);
  }
}

// out[t][:] = yshared[t][:] + sum_j ybuf[slot(t,j)][:], in bf16.
// Fixed summation order, so the result is deterministic.
// KT: top-k known at compile time (1..kMaxTopK), so the token's k rows are
// loaded together without spending registers on unused slots.
template <int KT>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  pdl_wait_and_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int d4 = a.d / 4;
  const int t = (int)(gid / d4), c = (int)(gid % d4);
  if (t >= a.T) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.yshared) acc = reinterpret_cast<const float4 *>(a.yshared + (size_t)t * a.d)[c];
  int slot[KT];
#pragma unroll
  for (int j = 0; j < KT; ++j) slot[j] = __ldg(a.slot_of_pair + t * KT + j);
  // the token's k rows in flight together, summed in slot order
  float4 v[KT];
#pragma unroll
  for (int j = 0; j < KT; ++j) v[j] = reinterpret_cast<const float4 *>(a.ybuf + (size_t)slot[j] * a.d)[c];
#pragma unroll
  for (int j = 0; j < KT; ++j) {
    acc.x += v[j].x; acc.y += v[j].y; acc.z += v[j].z; acc.w += v[j].w;
  }
  __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(a.out + (size_t)t * a.d + c * 4);
  o[0] = __floats2bfloat162_rn(acc.x, acc.y);
  o[1] = __floats2bfloat162_rn(acc.z, acc.w);
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t stream) {
  const unsigned grid = (unsigned)(((long long)a.T * (a.d / 4) + 255) / 256);
  if (grid == 0) return cudaSuccess;
  switch (a.k) {
#define TQ_COMBINE_K(K) \
  case K: return launch_pdl(combine_kernel<K>, dim3(grid), dim3(256), 0, stream, a);
    TQ_COMBINE_K(1) TQ_COMBINE_K(2) TQ_COMBINE_K(3) TQ_COMBINE_K(4)
    TQ_COMBINE_K(5) TQ_COMBINE_K(6) TQ_COMBINE_K(7) TQ_COMBINE_K(8)
#undef TQ_COMBINE_K
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// xs[slot][:] = w_slot * x16[token(slot)][:]  (fp16), for the linear layer.
__global__ void scale_gather_kernel(ScaleGatherArgs a) {
  pdl_wait_and_release();
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int d2 = a.d / 2;
  const int s = (int)(gid / d2), c = (int)(gid % d2);
  if (s >= a.P) return;
  const float w = a.slot_w[s];
  const __half2 v = reinterpret_cast<const __half2 *>(a.x16 + (size_t)a.slot_tok[s] * a.d)[c];
  const float2 f = __half22float2(v);
  reinterpret_cast<__half2 *>(a.xs + (size_t)s * a.ld)[c] = __floats2half2_rn(w * f.x, w * f.y);
}

// h[slot][f] = w_slot * silu(g) * u  (unfused path: activation after the per-expert adds)
__global__ void swiglu_kernel(SwigluArgs a) {
  pdl_wait_and_release();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n) return;
  const int slot = (int)(i / a.F), f = (int)(i % a.F);
  a.h[(size_t)slot * a.ldh + f] = half_checked(a.slot_w[slot] * silu_f(a.g[i]) * a.u[i], a.status);
}

// Bounded wait on an mbarrier that nothing arrives on: gives up after
// max_polls polls and records TILEQ_ERR_TIMEOUT.  Exercises the same bounded
// wait the pipelined kernels use, without any chance of a hang.
__global__ void bounded_wait_kernel(int *status, int max_polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t addr = smem_addr(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(addr) : "memory");
  uint32_t done = 0;
  for (int i = 0; i < max_polls && !done; ++i) {
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr)
        : "memory");
  }
  if (!done) set_status(status, TILEQ_ERR_TIMEOUT);
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];\n" ::"r"(addr) : "memory");
}

}  // namespace tileq
