// Closed-form centred affine fit of the linear stage's output correction.
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
// section "A closed-form fit avoids retraining from scratch": teacher (dense
// softmax) outputs and converted linear outputs are accumulated across scenes,
// tokens, heads and views, and a centred affine correction is fitted by a
// regularised least-squares solve in float64.
//
// Samples are pairs (x, y) of 64-vectors: x the linear stage's output before
// the correction, y the teacher's output, one pair per (token, head) of every
// call. Raw moments accumulate in float64 (count, sum x, sum y, sum x x^T,
// sum x y^T, sum |y|^2), per head or pooled over heads; the solve forms the centred
// covariances C_xx = E[x x^T] - mu_x mu_x^T, C_xy = E[x y^T] - mu_x mu_y^T and
// returns A^T = (C_xx + lam I)^-1 C_xy, b = mu_y - A mu_x.
//
//   affine_moments_kernel  CTA = (head, token chunk), 256 threads; 32-token
//                          tiles of x and y staged as doubles in shared memory;
//                          each thread owns a 4x4 block of sum x x^T and of
//                          sum x y^T (fp64 FMA); one partial per CTA.
//   affine_reduce_kernel   adds the partials of each group into the caller's
//                          moments in a fixed order (deterministic).
//   affine_solve_kernel    CTA = group: Cholesky factorisation of
//                          C_xx + lam I, forward and back substitution for the
//                          64 columns of A^T, all in fp64; fp32 A, b out.
//   affine_residual_kernel CTA = group: the mean |A x + b - y|^2 over the
//                          group's samples from its raw moments (the
//                          single-stage conversion error that ranks stages in
//                          section "Linear-centered stages plus tile-sparse
//                          stages").
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace zebra {

__device__ int g_affine_status;   // sticky: ZEBRA_ERR_NUMERIC when a solve met a non-positive pivot

int read_and_clear_affine_status(int* out) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_affine_status, sizeof(int)) != cudaSuccess) return ZEBRA_ERR_CUDA;
  const int z = 0;
  if (cudaMemcpyToSymbol(g_affine_status, &z, sizeof(int)) != cudaSuccess) return ZEBRA_ERR_CUDA;
  *out = v;
  return ZEBRA_OK;
}

constexpr int AF_TOK = 32;   // tokens per shared-memory tile

// 8 consecutive elements (16-byte aligned) as doubles
template <typename T>
__device__ __forceinline__ void load8(const T* p, double* d) {
  float f[8];
  load16(p, f);
  if (Elem<T>::PER16 == 4) load16(p + 4, f + 4);
#pragma unroll
  for (int e = 0; e < 8; ++e) d[e] = (double)f[e];
}

template <typename T>
__global__ void __launch_bounds__(256) affine_moments_kernel(const __grid_constant__ AffineArgs a) {
  __shared__ __align__(16) double xs[AF_TOK][AF_D];
  __shared__ __align__(16) double ys[AF_TOK][AF_D];
  const int tid = threadIdx.x;
  const int h = blockIdx.x, c = blockIdx.y;
  const long long n0 = (long long)c * a.chunk_tokens;
  const long long n1 = min(a.g.N, n0 + a.chunk_tokens);
  const T* X = static_cast<const T*>(a.x) + (long long)h * a.hs;
  const T* Y = static_cast<const T*>(a.y) + (long long)h * a.hs;
  const int ti = tid >> 4, tj = tid & 15;   // rows 4 ti .. 4 ti + 3, columns 4 tj .. 4 tj + 3
  double axx[4][4], axy[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) axx[i][j] = axy[i][j] = 0.0;
  double s1 = 0.0;   // threads 0-63: sum x[tid]; 64-127: sum y[tid - 64]
  for (long long nb = n0; nb < n1; nb += AF_TOK) {
    __syncthreads();   // the previous tile is consumed
    {
      const int tok = tid >> 3, part = tid & 7;   // 8 channels of one token per thread
      const long long n = nb + tok;
      double dx[8], dy[8];
      if (n < n1) {
        load8(X + n * a.ts + part * 8, dx);
        load8(Y + n * a.ts + part * 8, dy);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) dx[e] = dy[e] = 0.0;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        xs[tok][part * 8 + e] = dx[e];
        ys[tok][part * 8 + e] = dy[e];
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int tk = 0; tk < AF_TOK; ++tk) {
      double xi[4], xj[4], yj[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xi[e] = xs[tk][4 * ti + e];
        xj[e] = xs[tk][4 * tj + e];
        yj[e] = ys[tk][4 * tj + e];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          axx[i][j] = fma(xi[i], xj[j], axx[i][j]);
          axy[i][j] = fma(xi[i], yj[j], axy[i][j]);
        }
      if (tid < 64) s1 += xs[tk][tid];
      else if (tid < 128) s1 += ys[tk][tid - 64];
      else if (tid < 192) s1 = fma(ys[tk][tid - 128], ys[tk][tid - 128], s1);
    }
  }
  // sum |y|^2: threads 128-191 hold one channel each; two warp sums, then one add
  __shared__ double syy_w[2];
  if (tid >= 128 && tid < 192) {
    double v = s1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((tid & 31) == 0) syy_w[(tid - 128) >> 5] = v;
  }
  __syncthreads();
  double* part = a.part + ((size_t)h * a.chunks + c) * AF_STRIDE;
  if (tid == 0) {
    part[AF_N] = (double)(n1 > n0 ? n1 - n0 : 0);
    part[AF_SYY] = syy_w[0] + syy_w[1];
  }
  if (tid < 64) part[AF_SX + tid] = s1;
  else if (tid < 128) part[AF_SY + tid - 64] = s1;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = 4 * ti + i, q = 4 * tj + j;
      part[AF_SXX + r * AF_D + q] = axx[i][j];
      part[AF_SXY + r * AF_D + q] = axy[i][j];
    }
}

// moments[g] += sum of the partials of group g, in (head, chunk) order
__global__ void __launch_bounds__(256) affine_reduce_kernel(const __grid_constant__ AffineArgs a) {
  const int gidx = blockIdx.x;
  const int e = blockIdx.y * 256 + threadIdx.x;
  if (e >= AF_STRIDE) return;
  const int h0 = a.per_head ? gidx : 0, h1 = a.per_head ? gidx + 1 : a.g.H;
  double s = 0.0;
  for (int h = h0; h < h1; ++h)
    for (int c = 0; c < a.chunks; ++c) s += a.part[((size_t)h * a.chunks + c) * AF_STRIDE + e];
  a.moments[(size_t)gidx * AF_STRIDE + e] += s;
}

struct SolveSmem {
  double M[AF_D][AF_D];   // C_xx + lam I, then its Cholesky factor L (lower triangle)
  double R[AF_D][AF_D];   // C_xy, then Z = L^-1 C_xy, then W = A^T
  double mx[AF_D], my[AF_D];
  int bad;
};

__global__ void __launch_bounds__(256) affine_solve_kernel(const double* __restrict__ moments, int per_head, int heads,
                                                           double lam, float* __restrict__ A, float* __restrict__ b) {
  extern __shared__ __align__(16) unsigned char solve_raw[];
  SolveSmem& s = *reinterpret_cast<SolveSmem*>(solve_raw);
  const int tid = threadIdx.x, gidx = blockIdx.x;
  const double* m = moments + (size_t)gidx * AF_STRIDE;
  const double n = m[AF_N];
  if (tid == 0) s.bad = !(n > 0.0);
  if (tid < AF_D) {
    s.mx[tid] = n > 0.0 ? m[AF_SX + tid] / n : 0.0;
    s.my[tid] = n > 0.0 ? m[AF_SY + tid] / n : 0.0;
  }
  __syncthreads();
  for (int e = tid; e < AF_D * AF_D; e += 256) {
    const int i = e / AF_D, j = e - i * AF_D;
    const double inv = n > 0.0 ? 1.0 / n : 0.0;
    s.M[i][j] = m[AF_SXX + e] * inv - s.mx[i] * s.mx[j] + (i == j ? lam : 0.0);
    s.R[i][j] = m[AF_SXY + e] * inv - s.mx[i] * s.my[j];
  }
  __syncthreads();
  // Cholesky, right-looking: column k of L, then the trailing lower triangle
  for (int k = 0; k < AF_D; ++k) {
    if (tid == 0) {
      const double d = s.M[k][k];
      if (!(d > 0.0) || !isfinite(d)) {
        s.bad = 1;
        s.M[k][k] = 1.0;
      } else {
        s.M[k][k] = sqrt(d);
      }
    }
    __syncthreads();
    if (tid > k && tid < AF_D) s.M[tid][k] /= s.M[k][k];
    __syncthreads();
    const int w = AF_D - 1 - k;
    for (int e = tid; e < w * w; e += 256) {
      const int i = k + 1 + e / w, j = k + 1 + e % w;
      if (j <= i) s.M[i][j] -= s.M[i][k] * s.M[j][k];
    }
    __syncthreads();
  }
  if (tid < AF_D) {
    const int j = tid;   // column j of the right-hand side
    for (int i = 0; i < AF_D; ++i) {   // L Z = C_xy
      double z = s.R[i][j];
      for (int p = 0; p < i; ++p) z -= s.M[i][p] * s.R[p][j];
      s.R[i][j] = z / s.M[i][i];
    }
    for (int i = AF_D - 1; i >= 0; --i) {   // L^T W = Z
      double w = s.R[i][j];
      for (int p = i + 1; p < AF_D; ++p) w -= s.M[p][i] * s.R[p][j];
      s.R[i][j] = w / s.M[i][i];
    }
  }
  __syncthreads();
  const bool bad = s.bad != 0;
  if (bad && tid == 0) atomicExch(&g_affine_status, ZEBRA_ERR_NUMERIC);
  // A[j][i] = W[i][j]; b[j] = mu_y[j] - sum_i A[j][i] mu_x[i]
  const int h0 = per_head ? gidx : 0, h1 = per_head ? gidx + 1 : heads;
  for (int e = tid; e < AF_D * AF_D; e += 256) {
    const int j = e / AF_D, i = e - j * AF_D;
    const float v = bad ? __int_as_float(0x7fc00000) : (float)s.R[i][j];
    for (int h = h0; h < h1; ++h) A[((size_t)h * AF_D + j) * AF_D + i] = v;
  }
  if (tid < AF_D) {
    double acc = s.my[tid];
    for (int i = 0; i < AF_D; ++i) acc -= s.R[i][tid] * s.mx[i];
    const float v = bad ? __int_as_float(0x7fc00000) : (float)acc;
    for (int h = h0; h < h1; ++h) b[(size_t)h * AF_D + tid] = v;
  }
}

// Mean |A x + b - y|^2 of group g's samples from its raw moments:
//   sum |A x + b - y|^2 = tr(A Sxx A^T) + 2 b.(A sx) - 2 tr(A Sxy) + n |b|^2
//                         - 2 b.sy + sum |y|^2,
// divided by n (NaN for an empty group). A, b of the group: head g's when per
// head, head 0's when pooled. Fixed-order reductions (deterministic).
__global__ void __launch_bounds__(256) affine_residual_kernel(const double* __restrict__ moments, int per_head,
                                                              const float* __restrict__ A,
                                                              const float* __restrict__ b, double* __restrict__ err) {
  __shared__ double As[AF_D][AF_D + 1];
  __shared__ double bs[AF_D];
  __shared__ double part[256];
  const int tid = threadIdx.x, gidx = blockIdx.x;
  const double* m = moments + (size_t)gidx * AF_STRIDE;
  const int h = per_head ? gidx : 0;
  for (int e = tid; e < AF_D * AF_D; e += 256) As[e / AF_D][e % AF_D] = (double)A[(size_t)h * AF_D * AF_D + e];
  if (tid < AF_D) bs[tid] = (double)b[(size_t)h * AF_D + tid];
  __syncthreads();
  // thread (i = tid / 4, quarter = tid % 4) covers row i of A, columns q = quarter, quarter + 4, ...
  const int i = tid >> 2, qq = tid & 3;
  double acc = 0.0;
  for (int q = qq; q < AF_D; q += 4) {
    double u = 0.0;   // (A Sxx)[i][q]
    for (int p = 0; p < AF_D; ++p) u = fma(As[i][p], m[AF_SXX + p * AF_D + q], u);
    acc = fma(u, As[i][q], acc);                              // tr(A Sxx A^T)
    acc = fma(-2.0 * As[i][q], m[AF_SXY + q * AF_D + i], acc); // -2 tr(A Sxy)
    acc = fma(2.0 * bs[i] * As[i][q], m[AF_SX + q], acc);      // 2 b.(A sx)
  }
  if (qq == 0) acc += m[AF_N] * bs[i] * bs[i] - 2.0 * bs[i] * m[AF_SY + i];
  part[tid] = acc;
  __syncthreads();
  for (int w = 128; w >= 1; w >>= 1) {
    if (tid < w) part[tid] += part[tid + w];
    __syncthreads();
  }
  if (tid == 0) {
    const double n = m[AF_N];
    err[gidx] = n > 0.0 ? (part[0] + m[AF_SYY]) / n : __longlong_as_double(0x7ff8000000000000LL);
  }
}

int launch_affine_residual(const double* moments, int per_head, int heads, const float* A, const float* b,
                           double* err, cudaStream_t st) {
  const int groups = per_head ? heads : 1;
  {
    ProfScope prof("affine_residual", st);
    affine_residual_kernel<<<groups, 256, 0, st>>>(moments, per_head, A, b, err);
  }
  count_launch();
  return check_launch("affine_residual_kernel");
}

// chunks per head for the moments pass: about four CTAs per SM overall
int affine_chunks(const Geo& g) {
  const long long want = (4LL * 148 + g.H - 1) / g.H;
  const long long max_by_tokens = (g.N + AF_TOK - 1) / AF_TOK;
  long long c = want < max_by_tokens ? want : max_by_tokens;
  return (int)(c < 1 ? 1 : c);
}

template <typename T>
int launch_affine_moments(const AffineArgs& a, cudaStream_t st) {
  if (a.g.N == 0) return ZEBRA_OK;
  {
    ProfScope prof("affine_moments", st);
    affine_moments_kernel<T><<<dim3(a.g.H, a.chunks), 256, 0, st>>>(a);
  }
  count_launch();
  if (int rc = check_launch("affine_moments_kernel")) return rc;
  const int groups = a.per_head ? a.g.H : 1;
  {
    ProfScope prof("affine_reduce", st);
    affine_reduce_kernel<<<dim3(groups, (AF_STRIDE + 255) / 256), 256, 0, st>>>(a);
  }
  count_launch();
  return check_launch("affine_reduce_kernel");
}
template int launch_affine_moments<float>(const AffineArgs&, cudaStream_t);
template int launch_affine_moments<__nv_bfloat16>(const AffineArgs&, cudaStream_t);

int launch_affine_solve(const double* moments, int per_head, int heads, double lam, float* A, float* b,
                        cudaStream_t st) {
  const int groups = per_head ? heads : 1;
  cudaFuncSetAttribute(affine_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SolveSmem));
  {
    ProfScope prof("affine_solve", st);
    affine_solve_kernel<<<groups, 256, sizeof(SolveSmem), st>>>(moments, per_head, heads, lam, A, b);
  }
  count_launch();
  return check_launch("affine_solve_kernel");
}

}  // namespace zebra
