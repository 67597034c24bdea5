// Gaussian-sketch global low-rank decomposition of a projection's tiled matrix
// W_big [M*d_out, N*d_in] (expert k's bf16 weights in block (m, n) of the grid):
// TileQ summary, section 2.1, step 5 (global low-rank decomposition of W_big,
// approximated by Gaussian sketching instead of a full SVD).  The randomised
// range finder with an SVD of the projected matrix, computed as:
//
//   Y^T = Omega^T W_big^T                [l, R]   tcgen05 (bf16 in, fp32 out), W_big read by blocks
//   G   = Y^T Y                          [l, l]   fp64 accumulation
//   G   = E diag(lam) E^T                Jacobi, fp64: the rotations on one CTA (G in shared
//                                        memory), then E from the logged rotations, rows in parallel
//   Q^T = (E lam^-1/2)^T Y^T (lam > tol) [l, R]   orthonormal basis of range(Y), fp32
//   B   = Q^T W_big                      [l, C]   tcgen05 on the experts' transposes, Q^T
//                                                 split into two bf16 terms (hi + lo)
//   B B^T = Ub diag(s^2) Ub^T            Jacobi again
//   U  = Q Ub[:, :r],  Sigma = s[:r],  V = B^T Ub[:, :r] diag(1/s)
//
// so U diag(Sigma) V^T is the rank-r truncated SVD of Q Q^T W_big, the same
// quantity as the QR + SVD formulation.  The two eigen-decompositions of the
// small Gram matrices replace a tall QR and an SVD of B; both see fp64.
#include <cstring>

#include "kernels.cuh"

namespace tileq {
namespace {

constexpr int kSketchMaxL = TILEQ_SKETCH_MAX_L;  // sketch width: the l x l Gram matrix fits shared memory in fp64
constexpr int kSketchGramSplits = 16;             // row splits of a Gram matrix (partials summed in order)
constexpr double kSketchBasisTol = 1e-10;         // eigenvalues of Y^T Y below this times the largest are dropped

// ---------------------------------------------------------------- operands
// Element (i, k) of the left operand and (k, j) of the right one.
struct DenseF32 {
  const float *p;
  long long ld0, ld1;  // element (a, b) at p[a*ld0 + b*ld1]
  __device__ __forceinline__ float at(long long a, long long b) const { return p[a * ld0 + b * ld1]; }
};
// W_big (T = false) or its transpose (T = true), read blockwise from the
// experts' bf16 weights [K][d_out][d_in]; expert_of[m*N + n] is the expert in
// grid block (m, n).
template <bool T>
struct WBig {
  const __nv_bfloat16 *w;
  int N, d_out, d_in;
  int8_t expert_of[kMaxExperts];  // grid cell m*N + n -> expert
  __device__ __forceinline__ float at(long long a, long long b) const {
    const long long row = T ? b : a, col = T ? a : b;
    const int m = (int)(row / d_out), n = (int)(col / d_in);
    const int e = expert_of[m * N + n];
    return __bfloat162float(w[((size_t)e * d_out + (row - (long long)m * d_out)) * d_in + (col - (long long)n * d_in)]);
  }
};

// C[i][j] = cs[j] * sum_k A(i, k) B(k, j), fp32 accumulation.  64x64 tiles, K
// steps of 16 through shared memory, 4x4 outputs per thread.  A is loaded with
// consecutive threads along k (row-major W_big, dense row-major) or along i
// (transposed W_big), whichever is contiguous in memory.
constexpr int GT = 64, GK = 16;

template <typename AOp, bool A_ALONG_I>
__global__ void __launch_bounds__(256) sk_gemm_kernel(AOp A, DenseF32 B, float *C, long long ldc, int Mr, int Nc,
                                                      long long Kd, const float *cs) {
  __shared__ float as[GK][GT + 4];
  __shared__ float bs[GK][GT + 4];
  const int tid = threadIdx.x;
  const long long i0 = (long long)blockIdx.y * GT, j0 = (long long)blockIdx.x * GT;
  const int ti = (tid / 16) * 4, tj = (tid % 16) * 4;
  float acc[4][4] = {};
  for (long long k0 = 0; k0 < Kd; k0 += GK) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = tid + u * 256;  // 1024 elements of each 64 x 16 tile
      int ii, kk;
      if (A_ALONG_I) {
        ii = e % GT;
        kk = e / GT;
      } else {
        kk = e % GK;
        ii = e / GK;
      }
      const long long gi = i0 + ii, gk = k0 + kk;
      as[kk][ii] = (gi < Mr && gk < Kd) ? A.at(gi, gk) : 0.f;
      const int jj = e % GT, kb = e / GT;
      const long long gj = j0 + jj, gkb = k0 + kb;
      bs[kb][jj] = (gj < Nc && gkb < Kd) ? B.at(gkb, gj) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = as[kk][ti + u];
        b[u] = bs[kk][tj + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const long long gi = i0 + ti + u, gj = j0 + tj + v;
      if (gi < Mr && gj < Nc) C[gi * ldc + gj] = acc[u][v] * (cs ? cs[gj] : 1.f);
    }
}

// Gram partial: part[s][a][b] = sum over rows of split s of X[row][a] * X[row][b]
// in fp64 (X fp32 [rows][l]); one CTA per (32x32 tile of the l x l result, split).
constexpr int GR = 32;

__global__ void __launch_bounds__(256) sk_gram_kernel(const float *X, long long rows, int l, int splits,
                                                      double *part) {
  __shared__ float xa[GR][GR + 1];
  __shared__ float xb[GR][GR + 1];
  const int ta = blockIdx.x % ((l + GR - 1) / GR), tb = blockIdx.x / ((l + GR - 1) / GR);
  const int s = blockIdx.y;
  const long long per = (rows + splits - 1) / splits;
  const long long r0 = s * per, r1 = min(rows, r0 + per);
  const int a0 = ta * GR, b0 = tb * GR;
  const int tid = threadIdx.x;
  const int oa = tid / 8, ob = (tid % 8) * 4;  // this thread: row oa, columns ob..ob+3 of the tile
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (long long rr = r0; rr < r1; rr += GR) {
    for (int e = tid; e < GR * GR; e += 256) {
      const int rw = e / GR, c = e % GR;
      const long long row = rr + rw;
      xa[rw][c] = (row < r1 && a0 + c < l) ? X[row * l + a0 + c] : 0.f;
      xb[rw][c] = (row < r1 && b0 + c < l) ? X[row * l + b0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int rw = 0; rw < GR; ++rw) {
      const double va = xa[rw][oa];
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[v] += va * (double)xb[rw][ob + v];
    }
    __syncthreads();
  }
  double *out = part + (size_t)s * l * l;
#pragma unroll
  for (int v = 0; v < 4; ++v)
    if (a0 + oa < l && b0 + ob + v < l) out[(size_t)(a0 + oa) * l + b0 + ob + v] = acc[v];
}

// The same Gram partial of a row-major [l][rows] matrix (Y^T, B): rows along
// the contiguous dimension.
__global__ void __launch_bounds__(256) sk_gram_t_kernel(const float *Xt, long long rows, int l, int splits,
                                                        double *part) {
  __shared__ float xa[GR][GR + 1];
  __shared__ float xb[GR][GR + 1];
  const int ta = blockIdx.x % ((l + GR - 1) / GR), tb = blockIdx.x / ((l + GR - 1) / GR);
  const int s = blockIdx.y;
  const long long per = (rows + splits - 1) / splits;
  const long long r0 = s * per, r1 = min(rows, r0 + per);
  const int a0 = ta * GR, b0 = tb * GR;
  const int tid = threadIdx.x;
  const int oa = tid / 8, ob = (tid % 8) * 4;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (long long rr = r0; rr < r1; rr += GR) {
    for (int e = tid; e < GR * GR; e += 256) {
      const int c = e / GR, rw = e % GR;  // consecutive threads along the rows
      const long long row = rr + rw;
      xa[rw][c] = (row < r1 && a0 + c < l) ? Xt[(size_t)(a0 + c) * rows + row] : 0.f;
      xb[rw][c] = (row < r1 && b0 + c < l) ? Xt[(size_t)(b0 + c) * rows + row] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int rw = 0; rw < GR; ++rw) {
      const double va = xa[rw][oa];
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[v] += va * (double)xb[rw][ob + v];
    }
    __syncthreads();
  }
  double *out = part + (size_t)s * l * l;
#pragma unroll
  for (int v = 0; v < 4; ++v)
    if (a0 + oa < l && b0 + ob + v < l) out[(size_t)(a0 + oa) * l + b0 + ob + v] = acc[v];
}

// wt[k][c][r] = w[k][r][c] (bf16, 32 x 32 tiles through shared memory).
__global__ void sk_transpose_kernel(const __nv_bfloat16 *w, int d_out, int d_in, __nv_bfloat16 *wt) {
  __shared__ __nv_bfloat16 t[32][33];
  const int k = blockIdx.z;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const __nv_bfloat16 *src = w + (size_t)k * d_out * d_in;
  __nv_bfloat16 *dst = wt + (size_t)k * d_out * d_in;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < d_out && c < d_in) t[i][threadIdx.x] = src[(size_t)r * d_in + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < d_out && c < d_in) dst[(size_t)c * d_out + r] = t[threadIdx.x][i];
  }
}

// q (fp32) = hi + lo with hi = bf16(q), lo = bf16(q - hi): hl[0:n] = hi, hl[n:2n] = lo.
__global__ void sk_split_kernel(const float *q, long long n, __nv_bfloat16 *hl) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = q[i];
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  hl[i] = hi;
  hl[n + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// b[i] += b[n + i]: the hi and lo products summed.
__global__ void sk_sum_halves_kernel(float *b, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) b[i] += b[n + i];
}

// G[a][b] = sum of the splits' partials in split order.
__global__ void sk_gram_reduce_kernel(const double *part, int l, int splits, double *G) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= l * l) return;
  double v = 0.0;
  for (int s = 0; s < splits; ++s) v += part[(size_t)s * l * l + e];
  G[e] = v;
}

// Cyclic Jacobi eigen-decomposition of the symmetric l x l matrix G (fp64, l
// even, l <= kSketchMaxL).  Each round rotates l/2 disjoint index pairs of the
// round-robin schedule (index 0 fixed, the others rotating), the rotation of
// Golub and Van Loan's symmetric Schur step annihilating G[p][q]; sweeps of
// l-1 rounds until the off-diagonal mass is below (1e-13 ||G||)^2 or
// kJacobiSweeps sweeps.  One CTA applies the rotations to G, which lives in
// shared memory with a row stride of l + 1 (its columns are read too), and
// logs each round's (c, s, p, q); the eigenvectors E = J_1 J_2 ... are then
// formed from the log by sk_jacobi_vectors_kernel, whose rows are independent
// (a rotation of columns p, q of E changes each row on its own), so they run
// in parallel instead of adding a global-memory round trip to every round.
// lam[i] = the i-th largest eigenvalue and perm[i] the row of Et (= E^T)
// holding its eigenvector.
constexpr int kJacobiSweeps = 40;
constexpr int kJacobiThreads = 1024;

__global__ void __launch_bounds__(kJacobiThreads) sk_jacobi_kernel(const double *Gin, int l, double *lam, int *perm,
                                                                  double *log_c, double *log_s, int *log_pq,
                                                                  int *n_rounds) {
  extern __shared__ double G[];  // [l][l + 1]
  __shared__ double rc[kSketchMaxL / 2], rs[kSketchMaxL / 2];
  __shared__ int rp[kSketchMaxL / 2], rq[kSketchMaxL / 2];
  __shared__ double red[32];
  __shared__ int done;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int h = l / 2, ld = l + 1;
  for (int e = tid; e < l * l; e += nt) G[(e / l) * ld + e % l] = Gin[e];
  if (tid == 0) done = 0;
  int rounds = 0;
  __syncthreads();
  auto block_sum = [&](double v) -> double {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) red[tid >> 5] = v;
    __syncthreads();
    double t = 0.0;
    if (tid < 32) {
      t = tid < (nt >> 5) ? red[tid] : 0.0;
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    }
    __syncthreads();
    return t;  // valid in warp 0
  };
  for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
    // convergence: off-diagonal mass against the Frobenius mass
    double off = 0.0, all = 0.0;
    for (int e = tid; e < l * l; e += nt) {
      const double g = G[(e / l) * ld + e % l];
      all += g * g;
      if (e / l != e % l) off += g * g;
    }
    const double off_s = block_sum(off);
    const double all_s = block_sum(all);
    if (tid == 0) done = !(off_s > 1e-26 * all_s);
    __syncthreads();
    if (done) break;
    for (int t = 0; t < l - 1; ++t) {
      if (tid < h) {
        // round-robin pair i: positions i and l-1-i of [0, rotation of 1..l-1]
        auto player = [&](int pos) {
          if (pos == 0) return 0;
          const int v = pos - 1 + t;  // < 2 (l - 1)
          return (v >= l - 1 ? v - (l - 1) : v) + 1;
        };
        int p = player(tid), q = player(l - 1 - tid);
        if (p > q) {
          const int x = p;
          p = q;
          q = x;
        }
        // the symmetric Schur rotation annihilating G[p][q], in the form with
        // one division: t = 2 a sign(d) / (|d| + sqrt(d^2 + 4 a^2)), d = G[q][q] - G[p][p]
        const double apq = G[p * ld + q];
        double c = 1.0, sn = 0.0;
        if (apq != 0.0) {
          const double d = G[q * ld + q] - G[p * ld + p];
          const double tt = (d >= 0.0 ? 2.0 : -2.0) * apq / (fabs(d) + sqrt(d * d + 4.0 * apq * apq));
          c = rsqrt(1.0 + tt * tt);
          sn = tt * c;
        }
        rc[tid] = c;
        rs[tid] = sn;
        rp[tid] = p;
        rq[tid] = q;
        const size_t at = (size_t)rounds * h + tid;
        log_c[at] = c;
        log_s[at] = sn;
        log_pq[at] = p | (q << 16);
      }
      ++rounds;
      __syncthreads();
      // G <- J^T G J in one pass: the pairs partition the indices, so every
      // 2 x 2 block (rows p_i, q_i; columns p_j, q_j) becomes J_i^T G_ij J_j on its own
      for (int b = tid; b < h * h; b += nt) {
        const int bi = b / h, bj = b - bi * h;
        const int pi = rp[bi], qi = rq[bi], pj = rp[bj], qj = rq[bj];
        const double ci = rc[bi], si = rs[bi], cj = rc[bj], sj = rs[bj];
        const double g00 = G[pi * ld + pj], g01 = G[pi * ld + qj], g10 = G[qi * ld + pj], g11 = G[qi * ld + qj];
        // rows: [c -s; s c] applied as in the two-pass form (row p <- c p - s q, row q <- s p + c q)
        const double r00 = ci * g00 - si * g10, r01 = ci * g01 - si * g11;
        const double r10 = si * g00 + ci * g10, r11 = si * g01 + ci * g11;
        // columns: column p <- c p - s q, column q <- s p + c q
        G[pi * ld + pj] = cj * r00 - sj * r01;
        G[pi * ld + qj] = sj * r00 + cj * r01;
        G[qi * ld + pj] = cj * r10 - sj * r11;
        G[qi * ld + qj] = sj * r10 + cj * r11;
      }
      __syncthreads();
    }
  }
  // descending order of the eigenvalues; equal ones keep their index order
  for (int i = tid; i < l; i += nt) {
    const double li = G[i * ld + i];
    int rank = 0;
    for (int j = 0; j < l; ++j) {
      const double lj = G[j * ld + j];
      rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    lam[rank] = li;
    perm[rank] = i;
  }
  if (tid == 0) *n_rounds = rounds;
}

// E = J_1 J_2 ... J_n from the rotation log, written transposed (Et[q][j] =
// E[j][q]).  A CTA holds `rpb` rows of E in shared memory, starting from the
// identity; in every round its thread (pair i, row r) rotates entries p_i, q_i
// of row r (the round's pairs are disjoint), with the same arithmetic as a
// column rotation of E.  The next round's (c, s, p, q) is loaded before the
// round's barrier.
__global__ void __launch_bounds__(1024) sk_jacobi_vectors_kernel(const double *log_c, const double *log_s,
                                                               const int *log_pq, const int *n_rounds, int l, int rpb,
                                                               double *Et) {
  extern __shared__ double Er[];  // [rpb][l]
  const int h = l / 2, tid = threadIdx.x;
  const int row0 = blockIdx.x * rpb;
  const int rows = min(rpb, l - row0);
  for (int e = tid; e < rows * l; e += blockDim.x) Er[e] = (row0 + e / l == e % l) ? 1.0 : 0.0;
  const int i = tid % h, r = tid / h;
  const bool active = r < rows;
  const int nr = *n_rounds;
  double c = 0.0, sn = 0.0;
  int pq = 0;
  if (nr > 0) {
    c = log_c[i];
    sn = log_s[i];
    pq = log_pq[i];
  }
  __syncthreads();
  for (int t = 0; t < nr; ++t) {
    double cn = 0.0, snn = 0.0;
    int pqn = 0;
    if (t + 1 < nr) {
      const size_t at = (size_t)(t + 1) * h + i;
      cn = log_c[at];
      snn = log_s[at];
      pqn = log_pq[at];
    }
    if (active) {
      const int p = pq & 0xFFFF, q = pq >> 16;
      double *er = Er + r * l;
      const double ep = er[p], eq = er[q];
      er[p] = c * ep - sn * eq;
      er[q] = sn * ep + c * eq;
    }
    __syncthreads();
    c = cn;
    sn = snn;
    pq = pqn;
  }
  for (int e = tid; e < rows * l; e += blockDim.x) Et[(size_t)(e % l) * l + row0 + e / l] = Er[e];
}

// Wsmall[j][i] = E[j][perm[i]] / sqrt(lam[i]) for eigenvalues above tol * lam[0]
// (an orthonormal basis Q = Y Wsmall of range(Y)), zero columns otherwise.
__global__ void sk_basis_kernel(const double *Et, const double *lam, const int *perm, int l, double tol,
                                float *Wsmall) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= l * l) return;
  const int j = e / l, i = e % l;
  const double li = lam[i];
  Wsmall[e] = (li > tol * lam[0] && li > 0.0) ? (float)(Et[(size_t)perm[i] * l + j] / sqrt(li)) : 0.f;
}

// Ur[j][i] = E[j][perm[i]] (i < r), sigma[i] = sqrt(lam[i]), inv_sigma[i] = 1/sigma[i] (0 if sigma = 0).
__global__ void sk_select_kernel(const double *Et, const double *lam, const int *perm, int l, int r, float *Ur,
                                 float *sigma, float *inv_sigma) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < l * r) {
    const int j = e / r, i = e % r;
    Ur[e] = (float)Et[(size_t)perm[i] * l + j];
  }
  if (e < r) {
    const double s = sqrt(fmax(lam[e], 0.0));
    sigma[e] = (float)s;
    inv_sigma[e] = s > 0.0 ? (float)(1.0 / s) : 0.f;
  }
}

template <typename AOp, bool A_ALONG_I>
cudaError_t gemm(const AOp &A, const DenseF32 &B, float *C, long long ldc, long long Mr, int Nc, long long Kd,
                 const float *cs, cudaStream_t st) {
  const dim3 grid((unsigned)((Nc + GT - 1) / GT), (unsigned)((Mr + GT - 1) / GT));
  sk_gemm_kernel<AOp, A_ALONG_I><<<grid, 256, 0, st>>>(A, B, C, ldc, (int)Mr, Nc, Kd, cs);
  count_launches();
  return cudaGetLastError();
}

cudaError_t gram(const float *X, bool xt, long long rows, int l, double *part, int splits, double *G,
                 cudaStream_t st) {
  const int tiles = ((l + GR - 1) / GR) * ((l + GR - 1) / GR);
  if (xt)
    sk_gram_t_kernel<<<dim3(tiles, splits), 256, 0, st>>>(X, rows, l, splits, part);
  else
    sk_gram_kernel<<<dim3(tiles, splits), 256, 0, st>>>(X, rows, l, splits, part);
  count_launches();
  sk_gram_reduce_kernel<<<(l * l + 255) / 256, 256, 0, st>>>(part, l, splits, G);
  count_launches();
  return cudaGetLastError();
}

cudaError_t jacobi(const double *G, int l, double *E, double *lam, int *perm, double *log_c, double *log_s,
                   int *log_pq, int *n_rounds, cudaStream_t st) {
  const int smem = l * (l + 1) * (int)sizeof(double);
  static int configured = 0;
  if (smem > configured) {
    const int most = kSketchMaxL * (kSketchMaxL + 1) * (int)sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(sk_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    configured = most;
  }
  sk_jacobi_kernel<<<1, kJacobiThreads, smem, st>>>(G, l, lam, perm, log_c, log_s, log_pq, n_rounds);
  count_launches();
  const int h = l / 2;
  const int rpb = 1024 / h < 16 ? 1024 / h : 16;  // rows of E per CTA
  sk_jacobi_vectors_kernel<<<(l + rpb - 1) / rpb, h * rpb, (size_t)rpb * l * sizeof(double), st>>>(
      log_c, log_s, log_pq, n_rounds, l, rpb, E);
  count_launches();
  return cudaGetLastError();
}

// out[item][o] = sum_k A(o, k) Bop[item][k] on tcgen05 (bf16 operands, fp32 out):
// A is the grid of expert blocks in `a_arr` ([K][blk_rows][kblk], block of cell
// bi * cell_i + bk * cell_k), Bop the row-major bf16 [items][kd] matrix.
cudaError_t tc_grid_product(const __nv_bfloat16 *a_arr, int K, int blk_rows, int kblk, int grid_i, int cell_i,
                            int cell_k, const int8_t *blk_of, const __nv_bfloat16 *bop, int items, long long rows,
                            long long kd, float *out, cudaStream_t st) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  const int m_blocks = (int)(rows / 128);
  const int mb = m_blocks > 1 ? 2 : 1;
  a.pair = 0;
  a.m_blocks = m_blocks;
  a.m_units = (m_blocks + mb - 1) / mb;
  const int bn = dense_tile_items(items, a.m_units);
  if (!tensor_map_2b(&a.amap[0], a_arr, K * blk_rows, kblk, kblk, 128)) return cudaErrorInvalidValue;
  if (!tensor_map_2b(&a.bmap, bop, items, (int)kd, (int)kd, bn)) return cudaErrorInvalidValue;
  a.static_items = items;
  a.kblk = kblk;
  a.blk_rows = blk_rows;
  a.cell_i = cell_i;
  a.cell_k = cell_k;
  a.grid_i = grid_i;
  std::memcpy(a.a_blk, blk_of, kMaxExperts);
  a.bf16 = 1;
  a.d_out = (int)rows;
  a.d_in = (int)kd;
  a.epi = EPI_STORE_F32;
  a.out[0] = out;
  a.ldo = (int)rows;
  a.status = nullptr;
  const long long units = (long long)((items + bn - 1) / bn) * a.m_units;
  const int grid = (int)(units < 148 ? units : 148);
  return launch_gemm_dense(a, mb, bn, grid, st);
}

}  // namespace

// Workspace layout of the sketch (byte offsets, 256-byte aligned).
struct SketchWs {
  size_t wt, yt, qt, qhl, bo, part, g, e, lam, perm, wsmall, ur, inv_sigma, log_c, log_s, log_pq, n_rounds, total;
};

static size_t sk_align(size_t x) { return (x + 255) / 256 * 256; }

static SketchWs sketch_ws(int K, long long R, long long C, int d_out, int d_in, int l, int r) {
  SketchWs w{};
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += sk_align(b > 0 ? b : 16);
    return o;
  };
  w.wt = take((size_t)K * d_out * d_in * 2);
  w.yt = take((size_t)l * R * 4);
  w.qt = take((size_t)l * R * 4);
  w.qhl = take((size_t)2 * l * R * 2);
  w.bo = take((size_t)2 * l * C * 4);
  w.part = take((size_t)kSketchGramSplits * l * l * 8);
  w.g = take((size_t)l * l * 8);
  w.e = take((size_t)l * l * 8);
  w.lam = take((size_t)l * 8);
  w.perm = take((size_t)l * 4);
  w.wsmall = take((size_t)l * l * 4);
  w.ur = take((size_t)l * r * 4);
  w.inv_sigma = take((size_t)r * 4);
  // the rotation log of one Jacobi solve: at most kJacobiSweeps sweeps of l - 1 rounds of l/2 pairs
  const size_t log_n = (size_t)kJacobiSweeps * (l - 1) * (l / 2);
  w.log_c = take(log_n * 8);
  w.log_s = take(log_n * 8);
  w.log_pq = take(log_n * 4);
  w.n_rounds = take(4);
  w.total = off;
  return w;
}

static tileq_status sketch_check(const tileq_wbig *wb, int l, int r) {
  if (!wb || !wb->w || !wb->grid_assign) return TILEQ_ERR_INVALID_ARG;
  if (wb->M <= 0 || wb->N <= 0 || wb->K != wb->M * wb->N || wb->K > kMaxExperts) return TILEQ_ERR_UNSUPPORTED;
  if (wb->d_out <= 0 || wb->d_in <= 0) return TILEQ_ERR_INVALID_ARG;
  if (wb->d_out % 128 || wb->d_in % 128) return TILEQ_ERR_UNSUPPORTED;  // 128-row tiles of W_big and W_big^T
  if (l < 2 || l > kSketchMaxL || (l & 1) || r < 1 || r > l) return TILEQ_ERR_UNSUPPORTED;
  bool seen[kMaxExperts] = {};
  for (int k = 0; k < wb->K; ++k) {
    const int c = wb->grid_assign[k];
    if (c < 0 || c >= wb->K || seen[c]) return TILEQ_ERR_INVALID_ARG;
    seen[c] = true;
  }
  return TILEQ_OK;
}

}  // namespace tileq

using namespace tileq;

extern "C" tileq_status tileq_sketch_workspace_size(const tileq_wbig *wb, int l, int r, size_t *bytes) {
  if (!bytes) return TILEQ_ERR_INVALID_ARG;
  const tileq_status st = sketch_check(wb, l, r);
  if (st != TILEQ_OK) return st;
  *bytes = sketch_ws(wb->K, (long long)wb->M * wb->d_out, (long long)wb->N * wb->d_in, wb->d_out, wb->d_in, l, r).total;
  return TILEQ_OK;
}

extern "C" tileq_status tileq_sketch_lowrank(const tileq_wbig *wb, const void *omega_t, int l, int r, float *U,
                                             float *sigma, float *V, void *ws, size_t ws_bytes,
                                             tileq_stream_t stream_) {
  tileq_status st = sketch_check(wb, l, r);
  if (st != TILEQ_OK) return st;
  if (!omega_t || !U || !sigma || !V || !ws) return TILEQ_ERR_INVALID_ARG;
  const int M = wb->M, N = wb->N, K = wb->K, d_out = wb->d_out, d_in = wb->d_in;
  const long long R = (long long)M * d_out, C = (long long)N * d_in;
  const SketchWs w = sketch_ws(K, R, C, d_out, d_in, l, r);
  if (ws_bytes < w.total) return TILEQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream_);
  char *base = static_cast<char *>(ws);
  const __nv_bfloat16 *W = static_cast<const __nv_bfloat16 *>(wb->w);
  __nv_bfloat16 *Wt = reinterpret_cast<__nv_bfloat16 *>(base + w.wt);
  float *Yt = reinterpret_cast<float *>(base + w.yt);
  float *Qt = reinterpret_cast<float *>(base + w.qt);
  __nv_bfloat16 *Qhl = reinterpret_cast<__nv_bfloat16 *>(base + w.qhl);
  float *Bo = reinterpret_cast<float *>(base + w.bo);
  double *part = reinterpret_cast<double *>(base + w.part);
  double *G = reinterpret_cast<double *>(base + w.g);
  double *E = reinterpret_cast<double *>(base + w.e);
  double *lam = reinterpret_cast<double *>(base + w.lam);
  int *perm = reinterpret_cast<int *>(base + w.perm);
  float *Wsmall = reinterpret_cast<float *>(base + w.wsmall);
  float *Ur = reinterpret_cast<float *>(base + w.ur);
  float *inv_sigma = reinterpret_cast<float *>(base + w.inv_sigma);
  double *log_c = reinterpret_cast<double *>(base + w.log_c);
  double *log_s = reinterpret_cast<double *>(base + w.log_s);
  int *log_pq = reinterpret_cast<int *>(base + w.log_pq);
  int *n_rounds = reinterpret_cast<int *>(base + w.n_rounds);
  int8_t cell_expert[kMaxExperts] = {};
  for (int k = 0; k < K; ++k) cell_expert[wb->grid_assign[k]] = (int8_t)k;

#define SK(call)                                          \
  do {                                                    \
    if ((call) != cudaSuccess) return TILEQ_ERR_CUDA;     \
  } while (0)
  // Y^T = Omega^T W_big^T: output rows = rows of W_big (blocks of d_out, grid
  // row m), K = columns of W_big (blocks of d_in, grid column n)
  SK(tc_grid_product(W, K, d_out, d_in, M, N, 1, cell_expert, static_cast<const __nv_bfloat16 *>(omega_t), l, R, C,
                     Yt, s));
  // orthonormal basis of range(Y) from the eigen-decomposition of Y^T Y
  SK(gram(Yt, true, R, l, part, kSketchGramSplits, G, s));
  SK(jacobi(G, l, E, lam, perm, log_c, log_s, log_pq, n_rounds, s));
  sk_basis_kernel<<<(l * l + 255) / 256, 256, 0, s>>>(E, lam, perm, l, kSketchBasisTol, Wsmall);
  count_launches();
  SK(cudaGetLastError());
  // Q^T[i][row] = sum_j Wsmall[j][i] Y^T[j][row]
  SK((gemm<DenseF32, true>(DenseF32{Wsmall, 1, l}, DenseF32{Yt, R, 1}, Qt, R, l, (int)R, l, nullptr, s)));
  // B = Q^T W_big with Q^T = hi + lo (bf16 each): products on the experts' transposes,
  // output rows = columns of W_big (blocks of d_in, grid column n), K = rows of
  // W_big (blocks of d_out, grid row m)
  sk_transpose_kernel<<<dim3((d_in + 31) / 32, (d_out + 31) / 32, K), dim3(32, 8), 0, s>>>(W, d_out, d_in, Wt);
  count_launches();
  sk_split_kernel<<<(unsigned)((l * R + 255) / 256), 256, 0, s>>>(Qt, (long long)l * R, Qhl);
  count_launches();
  SK(cudaGetLastError());
  SK(tc_grid_product(Wt, K, d_in, d_out, N, 1, N, cell_expert, Qhl, 2 * l, C, R, Bo, s));
  sk_sum_halves_kernel<<<(unsigned)((l * C + 255) / 256), 256, 0, s>>>(Bo, (long long)l * C);
  count_launches();
  SK(cudaGetLastError());
  // eigen-decomposition of B B^T
  SK(gram(Bo, true, C, l, part, kSketchGramSplits, G, s));
  SK(jacobi(G, l, E, lam, perm, log_c, log_s, log_pq, n_rounds, s));
  sk_select_kernel<<<(l * r + 255) / 256, 256, 0, s>>>(E, lam, perm, l, r, Ur, sigma, inv_sigma);
  count_launches();
  SK(cudaGetLastError());
  // U[row][i] = sum_j Q^T[j][row] Ur[j][i];  V[c][i] = sum_j B[j][c] Ur[j][i] / sigma[i]
  SK((gemm<DenseF32, true>(DenseF32{Qt, 1, R}, DenseF32{Ur, r, 1}, U, r, R, r, l, nullptr, s)));
  SK((gemm<DenseF32, true>(DenseF32{Bo, 1, C}, DenseF32{Ur, r, 1}, V, r, C, r, l, inv_sigma, s)));
#undef SK
  return TILEQ_OK;
}
