// Linear global attention with the per-head centered affine correction.
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views":
//  - section "Speedup scales with the number of input views": the linear-stage
//    kernels fuse Q/K normalisation, positional rotation and the channel-softmax
//    feature map;
//  - section "Linear-centered stages plus tile-sparse stages": linear-centered
//    attention aggregates global context at linear cost;
//  - section "A closed-form fit avoids retraining from scratch": a centered
//    affine correction is applied to each linear stage's output.
//
// Per head h: f(x) = phi(rope2d(rmsnorm(x))), S = sum_n f(k_n) v_n^T, z = sum_n f(k_n),
// y_n = A (S^T f(q_n)) / (z . f(q_n)) + b. Folding A into the state
// (S' = S A^T) makes the epilogue one 64x65 contraction per token.
//
// Three kernels:
//  1. state:  per (head, token chunk) CTA: K and V blocks by bulk tensor copies,
//     prologue on K in registers (4 threads per token, 16 channels each),
//     f(K) -> its own K ring stage as bf16, then
//     [S | z] += f(K)^T [V | ones] on the tcgen05 tensor cores (M = 64 channels,
//     N = 64 for S and 16 for z, K = 64 tokens per block, fp32 accumulators in
//     tensor memory; one thread issues, the next block's prologue overlaps),
//     fp32 partials per chunk.
//  2. reduce: per head, sums the chunk partials in a fixed order (deterministic),
//     forms S' = S A^T, and writes the bf16 B operand [S' | z] of the apply kernel.
//  3. apply:  per (head, token chunk) CTA: prologue on Q (f(Q) overwrites its
//     own ring stage; the softmax's division by its sum is left out, since it
//     cancels in the ratio below), f(Q) [S' | z] on the tcgen05 tensor cores
//     (M = 64 tokens, N = 72, accumulators in tensor memory), divide by the z
//     column, add b, stage the bf16 block by stmatrix and store it by one bulk
//     tensor copy.
// The fp32 variants run the same three steps with plain fp32 arithmetic.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace zebra {

constexpr int NB = 72;  // 64 state columns + z column, padded to a multiple of 8

__device__ __forceinline__ void token_pos(const Geo& g, long long n, bool& special, int& row, int& col) {
  const int j = (int)(n % g.L);
  special = j < g.S;
  const int p = j - g.S;
  row = special ? 0 : p / g.Wp;
  col = special ? 0 : p - (p / g.Wp) * g.Wp;
}

// Position j (0 <= j < L) of a token within its view: special token, or patch
// (row, col). Multiply-shift division; exact for every int32 j and divisor.
__device__ __forceinline__ void view_pos(const Geo& g, int j, bool& special, int& row, int& col) {
  special = j < g.S;
  const int p = special ? 0 : j - g.S;
  row = fdiv(p, g.fWp);
  col = p - row * g.Wp;
}
// j mod L for 0 <= j < 2^31
__device__ __forceinline__ int mod_L(const Geo& g, int j) { return j - fdiv(j, g.fL) * g.L; }
// j mod L for 0 <= j < L + 64: one compare and subtract when a view has at least 64 tokens
__device__ __forceinline__ int wrap_L(const Geo& g, int j) {
  if (g.L >= 64) return j >= g.L ? j - g.L : j;
  return mod_L(g, j);
}

// full 64-channel prologue in one thread (fp32 path)
__device__ __forceinline__ void features_full(float* x, bool special, int row, int col,
                                              const float2* __restrict__ tab, float eps) {
  float ss = 0.f;
  for (int c = 0; c < 64; ++c) ss = fmaf(x[c], x[c], ss);
  const float sc = 1.0f / sqrtf(ss * (1.0f / D) + eps);
  for (int c = 0; c < 64; ++c) x[c] *= sc;
  if (!special) {
    for (int half = 0; half < 2; ++half) {
      const int pos = half ? col : row;
      for (int j = 0; j < 16; ++j) {
        const float2 cs = tab[pos * 16 + j];
        const float a = x[32 * half + j], b = x[32 * half + j + 16];
        x[32 * half + j] = a * cs.x - b * cs.y;
        x[32 * half + j + 16] = b * cs.x + a * cs.y;
      }
    }
  }
  float mx = x[0];
  for (int c = 1; c < 64; ++c) mx = fmaxf(mx, x[c]);
  float sum = 0.f;
  for (int c = 0; c < 64; ++c) {
    x[c] = expf(x[c] - mx);
    sum += x[c];
  }
  for (int c = 0; c < 64; ++c) x[c] /= sum;
}

// --------------------------------------------------------------------------
// shared-memory addressing: 64 x 128-byte tiles with the 128-byte swizzle
// (16-byte chunk c of row r at chunk c ^ (r % 8))
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lsmem(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ uint32_t lswz(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }
// --------------------------------------------------------------------------
// 1/3. state and apply (bf16), four threads per token
// --------------------------------------------------------------------------
// Raw bf16 rows of a 64-token block, one 128-byte head slice per token, land in
// a ring of 128-byte-swizzled shared tiles, by bulk tensor copies where a tensor
// map describes the input layout, else by 16-byte asynchronous copies (rows past
// the tensor's end zero-filled either way): 3 stages of K and V in the state
// kernel, LA_STAGES of Q in the apply kernel, each refilled once the MMAs that
// read the block it held have completed and every warp has passed a barrier
// after its own use of it.
constexpr int LSTAGES = 3;
#ifndef ZEBRA_LIN_ASTAGES
#define ZEBRA_LIN_ASTAGES 3
#endif
constexpr int LA_STAGES = ZEBRA_LIN_ASTAGES;   // Q ring depth of the apply kernel

// State kernel shared memory (base aligned to 1024 bytes, like every tile in it):
// the K and V rings (f(K) overwrites its own K stage), the all-ones B operand of
// the z MMAs, the MMA completion barrier and the tensor-memory base.
struct StateSmem {
  unsigned char k[LSTAGES][64 * 128];
  unsigned char v[LSTAGES][64 * 128];
  unsigned char ones[16 * 128];
  uint64_t full[LSTAGES];   // K and V of a stage landed (bulk tensor copies)
  uint64_t mma_bar;
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t STATE_TMEM_COLS = 128;   // [S | z]: columns 0-63 and 64-79
// 4 CTAs per SM: shared memory (+ 1 KB base alignment, + 1 KB the system keeps per CTA) and TMEM
static_assert(4 * (sizeof(StateSmem) + 1024 + 1024) <= 228 * 1024, "four CTAs of the state kernel per SM");
static_assert(4 * STATE_TMEM_COLS <= 512, "four CTAs' tensor memory per SM");

// Bounded waits of the linear stage's tcgen05 kernels: the sticky status word,
// the wait limit, and the error-path test hook (the token block of each chunk
// whose MMAs the state kernel leaves out; -1 = none).
__device__ int g_lin_status;
__device__ unsigned long long g_lin_wait_ns = 2000000000ull;
__device__ int g_lin_inject_block = -1;

int set_linear_debug_inject(int block, unsigned long long wait_ns) {
  const int b = block < 0 ? -1 : block;
  const unsigned long long w = wait_ns ? wait_ns : 2000000000ull;
  if (cudaMemcpyToSymbol(g_lin_inject_block, &b, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_lin_wait_ns, &w, sizeof(w)) != cudaSuccess)
    return ZEBRA_ERR_CUDA;
  return ZEBRA_OK;
}

int read_and_clear_linear_status(int* out) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_lin_status, sizeof(int)) != cudaSuccess) return ZEBRA_ERR_CUDA;
  const int z = 0;
  if (cudaMemcpyToSymbol(g_lin_status, &z, sizeof(int)) != cudaSuccess) return ZEBRA_ERR_CUDA;
  *out = v;
  return ZEBRA_OK;
}

// The calling thread waits for the phase of `parity` of `b`; after
// g_lin_wait_ns it records ZEBRA_ERR_TIMEOUT and returns false.
__device__ __noinline__ bool lin_wait_slow(uint64_t* b, uint32_t parity) {
  const unsigned long long limit = *(volatile unsigned long long*)&g_lin_wait_ns;
  const unsigned long long t0 = tc::gtime();
  while (!tc::mbar_try(b, parity)) {
    if (tc::gtime() - t0 > limit) {
      atomicExch(&g_lin_status, ZEBRA_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// the first test inline (it suspends the thread until the phase completes or the hint runs out)
__device__ __forceinline__ bool lin_wait(uint64_t* b, uint32_t parity) {
  return tc::mbar_try(b, parity) || lin_wait_slow(b, parity);
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 256 threads, 64 tokens per step. Thread (tok = token_of(tid), part = tid % 4) owns
// 16 channels of its token that form 8 whole rotation pairs: half = part / 2
// (channels 0-31 turn by patch row, 32-63 by column), sub = part % 2 (pairs
// j = 8 sub .. 8 sub + 7 of the half): the "a" channels 32 half + 8 sub .. + 7
// and their partners 16 further. The four threads of a token combine the RMS
// norm and the sum with two shuffles each. The contractions run on the tensor
// cores; to read an accumulator back, warp w takes rows 16 (w % 4) .. + 15 (its
// tensor-memory lane quarter) and columns 32 (w / 4) .. + 31.
constexpr int LQ_THREADS = 256;
// Token of thread tid: the quads of a warp take its 8 tokens in the order 0 2 1 3 4 6 5 7,
// so the two tokens of each 8-lane phase of a 16-byte shared access are rows r and r + 2.
// Their chunk sets {0 1 4 5} and {2 3 6 7} (before the swizzle's XOR with the row) are
// disjoint, and the reads, writes and copies of the rows are free of bank conflicts.
__device__ __forceinline__ int token_of(int tid) {
  const int q = (tid >> 2) & 7;
  return (tid >> 5) * 8 + ((q & 4) | ((q & 1) << 1) | ((q >> 1) & 1));
}

// This thread's part of its token's row in one tensor: two 16-byte pieces per
// 64-token block (the "a" channels and, 2 chunks on, their partners), copied
// into a ring stage at the fixed swizzled offsets oa, ob. The source walks
// down the chunk by 64 token rows per fetched block; pieces of rows past the
// chunk's end are zero-filled (read from the tensor's base, never past it).
struct RowFetch {
  const __nv_bfloat16* base;
  const __nv_bfloat16* p;   // this thread's row in the next block to fetch
  long long step;           // 64 token rows
  __device__ __forceinline__ RowFetch(const __nv_bfloat16* t, long long n0, long long ts, int tok, int half, int sub)
      : base(t), p(t + (n0 + tok) * ts + 32 * half + 8 * sub), step(64 * ts) {}
  __device__ __forceinline__ void fetch(uint32_t stage, uint32_t oa, uint32_t ob, bool ok) {
    const __nv_bfloat16* src = ok ? p : base;
    const int n = ok ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(stage + oa), "l"(src), "r"(n));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(stage + ob), "l"(src + 16), "r"(n));
    p += step;
  }
};

// Packed fp32 pairs (sm_100 f32x2 arithmetic): two lanes of work per instruction.
// Inline PTX rather than the __ffma2_rn family: with those the state kernel
// spilled and ran 3% slower.
__device__ __forceinline__ float2 l_fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2,%3};\n mov.b64 rb, {%4,%5};\n mov.b64 rc, {%6,%7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0,%1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 l_mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2,%3};\n mov.b64 rb, {%4,%5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0,%1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 l_add2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2,%3};\n mov.b64 rb, {%4,%5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0,%1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 l_sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2,%3};\n mov.b64 rb, {%4,%5};\n"
      " sub.rn.f32x2 rd, ra, rb;\n mov.b64 {%0,%1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// f(x) on this thread's 16 channels (xa: the "a" channels of its 8 rotation
// pairs, xb: their partners), the elementwise steps on f32x2 pairs (channels
// 2p, 2p + 1 of xa and of xb). It rests on three facts:
//  - the rotation keeps the norm of each pair, so the RMS scale sc of the raw
//    channels is that of the rotated ones, and, the rotation being linear, sc
//    goes into the exponent: exp(sc r_c) = exp2(r_c (sc log2 e));
//  - every channel of sc x has |sc x_c| <= sqrt(64) = 8 (the RMS of the 64
//    channels is at most 1), so exp(sc r_c) lies in [e^-8, e^8] and the
//    channel softmax needs no maximum shift;
//  - with NORMALISE = false the division by the sum is left out: the apply
//    kernel's output is a ratio of two contractions that are both linear in
//    f(q), so the sum cancels.
// The sum of squares goes across the token's 4 threads while the rotation runs.
// Padding tokens (valid = false, zero-filled) get exponent arguments 0 and,
// when normalised, features 0.
template <bool NORMALISE>
__device__ __forceinline__ void features_lin(float* xa, float* xb, int half, int sub, bool special, int row, int col,
                                             const float4* __restrict__ tab, int maxpos, float eps, bool valid) {
  float2* A = reinterpret_cast<float2*>(xa);
  float2* B = reinterpret_cast<float2*>(xb);
  float2 s0 = l_mul2(A[0], A[0]), s1 = l_mul2(A[1], A[1]);
  s0 = l_fma2(A[2], A[2], s0);
  s1 = l_fma2(A[3], A[3], s1);
  s0 = l_fma2(B[0], B[0], s0);
  s1 = l_fma2(B[1], B[1], s1);
  s0 = l_fma2(B[2], B[2], s0);
  s1 = l_fma2(B[3], B[3], s1);
  s0 = l_add2(s0, s1);
  float ss = s0.x + s0.y;
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  if (!special) {
    // pair group 4 sub + p at the half's position: (cos, cos', sin, sin'). Consecutive
    // tokens of a warp read consecutive positions of a group: few L1 lines per load.
    const float4* t = tab + 4 * sub * maxpos + (half ? col : row);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float4 cs = __ldg(t + p * maxpos);
      const float2 c = make_float2(cs.x, cs.y), sn = make_float2(cs.z, cs.w);
      const float2 a = A[p], b = B[p];
      A[p] = l_sub2(l_mul2(a, c), l_mul2(b, sn));   // a cos - b sin
      B[p] = l_fma2(b, c, l_mul2(a, sn));           // b cos + a sin
    }
  }
  const float k = valid ? rsqrtf(ss * (1.0f / D) + eps) * LOG2E : 0.f;
  const float2 k2 = make_float2(k, k);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 ea = l_mul2(A[p], k2), eb = l_mul2(B[p], k2);
    A[p] = make_float2(fast_exp2(ea.x), fast_exp2(ea.y));
    B[p] = make_float2(fast_exp2(eb.x), fast_exp2(eb.y));
  }
  if (NORMALISE) {
    float2 t0 = l_add2(l_add2(A[0], A[1]), l_add2(A[2], A[3]));
    const float2 t1 = l_add2(l_add2(B[0], B[1]), l_add2(B[2], B[3]));
    t0 = l_add2(t0, t1);
    float sum = t0.x + t0.y;
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    const float inv = valid ? __fdividef(1.0f, sum) : 0.f;   // sum lies in [64 e^-8, 64 e^8]
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      A[p] = l_mul2(A[p], inv2);
      B[p] = l_mul2(B[p], inv2);
    }
  }
}

__device__ __forceinline__ void read_q4(const unsigned char* tile, uint32_t oa, uint32_t ob, float* xa, float* xb) {
  const uint4 wa = *reinterpret_cast<const uint4*>(tile + oa);
  const uint4 wb = *reinterpret_cast<const uint4*>(tile + ob);
  const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&wa);
  const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&wb);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 fa = __bfloat1622float2(ha[e]), fb = __bfloat1622float2(hb[e]);
    xa[2 * e] = fa.x;
    xa[2 * e + 1] = fa.y;
    xb[2 * e] = fb.x;
    xb[2 * e + 1] = fb.y;
  }
}

__device__ __forceinline__ void store_q4(unsigned char* tile, uint32_t oa, uint32_t ob, const float* xa, const float* xb) {
  uint4 va, vb;
  __nv_bfloat162* ha = reinterpret_cast<__nv_bfloat162*>(&va);
  __nv_bfloat162* hb = reinterpret_cast<__nv_bfloat162*>(&vb);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    ha[e] = __floats2bfloat162_rn(xa[2 * e], xa[2 * e + 1]);
    hb[e] = __floats2bfloat162_rn(xb[2 * e], xb[2 * e + 1]);
  }
  *reinterpret_cast<uint4*>(tile + oa) = va;
  *reinterpret_cast<uint4*>(tile + ob) = vb;
}

__device__ __forceinline__ int ring_next(int s, int n) { return s + 1 == n ? 0 : s + 1; }

// [S | z] += f(K)^T [V | ones] of one 64-token block on the tensor cores: A = f(K)^T
// (MN-major: the K stage's rows are tokens, its 64 channels the M dimension),
// B = V (MN-major) for S (N = 64, TMEM columns 0-63) and the all-ones tile
// (K-major, N = 16) for z (columns 64-79); K = 16 tokens per MMA, 2,048 bytes of
// the stages per step. acc = 0 starts both accumulators. One elected lane of
// the warp issues the eight MMAs and the commit to `bar`.
__device__ __forceinline__ void state_mma_elect(uint32_t tmem, uint64_t fk, uint64_t v, uint64_t ones, uint32_t acc,
                                                uint64_t* bar) {
  constexpr uint32_t ID_S = tc::idesc(true, 64, true), ID_Z = tc::idesc(false, 16, true);
  asm volatile(
      "{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, %16, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %14, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %14, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %14, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %9, %14, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %2, %10, %15, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %3, %11, %15, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %4, %12, %15, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%1], %5, %13, %15, p1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%17];\n}\n"
      ::"r"(tmem), "r"(tmem + 64), "l"(fk), "l"(fk + 128), "l"(fk + 256), "l"(fk + 384), "l"(v), "l"(v + 128),
      "l"(v + 256), "l"(v + 384), "l"(ones), "l"(ones + 2), "l"(ones + 4), "l"(ones + 6), "r"(ID_S), "r"(ID_Z),
      "r"(acc), "r"(tc::saddr(bar))
      : "memory");
}

// Tensor maps of the state kernel's K and V inputs ([N, H, 64] strided by (ts, hs)): 3D maps with
// the channels innermost, the outer two dimensions in the order of their strides (head_outer = 0:
// {64, H, N}, coordinates (0, h, n); 1: {64, N, H}, coordinates (0, n, h)), a box of 64 channels x
// one head x 64 tokens and the 128-byte swizzle. Layouts a map cannot describe take the 16-byte
// asynchronous copies instead.
struct StateParams {
  CUtensorMap tk, tv;
  LinearArgs a;
  int head_outer;
};

__device__ __forceinline__ void l_tma_3d(uint32_t dst, const CUtensorMap* map, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(map), "r"(0), "r"(c1), "r"(c2), "r"(lsmem(bar))
      : "memory");
}

template <bool TMA_IN>
__global__ void __launch_bounds__(LQ_THREADS, 4) linear_state_q4_kernel(const __grid_constant__ StateParams prm) {
  extern __shared__ unsigned char state_smem_raw[];
  StateSmem& ss = *reinterpret_cast<StateSmem*>(align1024(state_smem_raw));
  const LinearArgs& a = prm.a;
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x;   // grid (head, chunk): the heads of the same tokens run together
  const long long n0 = (long long)blockIdx.y * a.chunk_tokens;
  const long long n1 = min((long long)g.N, n0 + a.chunk_tokens);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.k) + (long long)h * a.hs;
  const __nv_bfloat16* Vt = static_cast<const __nv_bfloat16*>(a.v) + (long long)h * a.hs;
  const int tok = token_of(tid), half = (tid >> 1) & 1, sub = tid & 1;

  const int nblk = (int)((n1 - n0 + 63) / 64);
  const int left = (int)(n1 - n0) - tok;   // block i holds this thread's token iff 64 i < left
  const uint32_t oa = lswz(tok, 4 * half + sub), ob = lswz(tok, 4 * half + sub + 2);
  const uint32_t kst = lsmem(ss.k[0]), vst = lsmem(ss.v[0]);
  RowFetch fk(K, n0, a.ts, tok, half, sub), fv(Vt, n0, a.ts, tok, half, sub);
  // block f into ring stage `stage`: one thread arms the stage's barrier and issues two bulk tensor
  // copies (rows past the tensor's end are zero-filled), or every thread copies its 16-byte pieces
  auto load = [&](int f, int stage) {
    if constexpr (TMA_IN) {
      if (tid == 0) {
        const int n = (int)(n0 + 64LL * f);
        const int c1 = prm.head_outer ? n : h, c2 = prm.head_outer ? h : n;
        tc::mbar_expect_tx(&ss.full[stage], 2 * 64 * 128);
        l_tma_3d(kst + stage * 8192, &prm.tk, c1, c2, &ss.full[stage]);
        l_tma_3d(vst + stage * 8192, &prm.tv, c1, c2, &ss.full[stage]);
      }
    } else {
      fk.fetch(kst + stage * 8192, oa, ob, 64 * f < left);
      fv.fetch(vst + stage * 8192, oa, ob, 64 * f < left);
    }
  };
  if (tid == 0) {
    tc::mbar_init(&ss.mma_bar, 1);
    for (int i = 0; i < LSTAGES; ++i) tc::mbar_init(&ss.full[i], 1);
    ss.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < 16 * 128 / 4; i += LQ_THREADS) reinterpret_cast<uint32_t*>(ss.ones)[i] = 0x3F803F80u;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the ones tile is read by the tensor cores
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(lsmem(&ss.tmem_base)),
                 "r"(STATE_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  for (int i = 0; i < LSTAGES - 1; ++i) {   // the barriers are initialised: the first blocks go out
    if (i < nblk) load(i, i);
    if constexpr (!TMA_IN) asm volatile("cp.async.commit_group;\n" ::);
  }
  const uint32_t tmem = ss.tmem_base;
  const uint64_t d_k0 = tc::desc_mn(kst), d_v0 = tc::desc_mn(vst), d_ones = tc::desc_k(lsmem(ss.ones));
  const int inject = *(volatile int*)&g_lin_inject_block;
  int issued = 0, waited = 0;   // thread 0: blocks whose MMAs went out / were seen complete
  int consumed = 0;             // blocks whose loop iteration ran to its end
  int jb = (int)(n0 % g.L);   // view position of the current block's first token
  int st = 0, fst = LSTAGES - 1;   // ring stages of block i and of block i + LSTAGES - 1
  for (int i = 0; i < nblk; ++i) {
    if constexpr (TMA_IN) {
      if (!lin_wait(&ss.full[st], (i / LSTAGES) & 1)) ss.abort = 1;
    } else {
      // Block i's copies are the oldest but LSTAGES - 2 groups in flight.
      asm volatile("cp.async.wait_group %0;\n" ::"n"(LSTAGES - 2));
    }
    __syncthreads();
    const bool valid = 64 * i < left;
    float xa[8], xb[8];
    read_q4(ss.k[st], oa, ob, xa, xb);
    {
      bool sp;
      int row, col;
      view_pos(g, wrap_L(g, jb + tok), sp, row, col);
      jb = wrap_L(g, jb + 64);
      features_lin<true>(xa, xb, half, sub, sp, row, col, a.rope_g, a.maxpos, a.eps, valid);
    }
    store_q4(ss.k[st], oa, ob, xa, xb);   // f(K) over its own K rows
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor cores
    // block i - 1's MMAs are done with their stages before block i + LSTAGES - 1 refills them
    if (tid == 0 && i > 0) {
      if (lin_wait(&ss.mma_bar, (i - 1) & 1))
        waited = i;
      else
        ss.abort = 1;
    }
    __syncthreads();
    if (ss.abort) break;
    if (warp == 0 && i != inject) {
      tc::fence_after();
      state_mma_elect(tmem, d_k0 + st * 512, d_v0 + st * 512, d_ones, i > 0 ? 1u : 0u, &ss.mma_bar);
      issued = i + 1;
    }
    {
      const int f = i + LSTAGES - 1;
      if (f < nblk) load(f, fst);
      if constexpr (!TMA_IN) asm volatile("cp.async.commit_group;\n" ::);
    }
    st = ring_next(st, LSTAGES);
    fst = ring_next(fst, LSTAGES);
    consumed = i + 1;
  }
  if constexpr (TMA_IN) {
    // after an abort, bulk copies that went out but were not waited for land first (bounded again)
    if (tid == 0 && ss.abort)
      for (int f = consumed; f < min(nblk, consumed + LSTAGES - 1); ++f)
        lin_wait(&ss.full[f % LSTAGES], (f / LSTAGES) & 1);
  } else {
    asm volatile("cp.async.wait_group 0;\n" ::);
  }
  if (tid == 0) {
    if (!ss.abort && nblk > 0) {   // the last block's MMAs
      if (lin_wait(&ss.mma_bar, (nblk - 1) & 1))
        waited = nblk;
      else
        ss.abort = 1;
    }
    // after an abort, MMAs that went out but were not seen complete land first (bounded again)
    if (ss.abort && issued > waited) lin_wait(&ss.mma_bar, (issued - 1) & 1);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (!ss.abort) {
    // warp w reads the M = 64 accumulator rows 16 (w % 4) .. + 15 from its TMEM lane quarter
    // (16x256b shape: rows g4 and g4 + 8, columns 2 q4 and 2 q4 + 1 of each 8), columns
    // 32 (w / 4) .. + 31, and warps 0-3 the z column 64
    const int quarter = warp & 3, cg = warp >> 2, g4 = lane >> 2, q4 = lane & 3;
    const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
    float r[16];
    tc::tmem_ld32(trow + 32 * cg, r);
    float* part = a.part + ((size_t)blockIdx.y * g.H + h) * 64 * 65;
    const int r0 = 16 * quarter + g4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 32 * cg + 8 * j + 2 * q4;
      part[r0 * 65 + c] = r[4 * j];
      part[r0 * 65 + c + 1] = r[4 * j + 1];
      part[(r0 + 8) * 65 + c] = r[4 * j + 2];
      part[(r0 + 8) * 65 + c + 1] = r[4 * j + 3];
    }
    if (cg == 0) {
      float z[4];
      tc::tmem_ld8(trow + 64, z);
      if (q4 == 0) {
        part[r0 * 65 + 64] = z[0];
        part[(r0 + 8) * 65 + 64] = z[2];
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(STATE_TMEM_COLS));
}

// Apply kernel shared memory: the Q ring, one output block, the B operand, the
// MMA completion barrier and the tensor-memory base. Every tile starts on a
// 1024-byte boundary, so the swizzled offsets lswz() are the 128-byte swizzle of
// the tensor cores' operand reads and of the bulk tensor copies.
struct ApplySmem {
  unsigned char q[LA_STAGES][64 * 128];
  unsigned char out[2][64 * 128];
  unsigned char b[NB * 128];
  uint64_t full[LA_STAGES];   // Q of a stage landed (bulk tensor copies)
  uint64_t mma_bar;
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t APPLY_TMEM_COLS = 128;   // f(Q) [S' | z]: columns 0-71
static_assert(4 * APPLY_TMEM_COLS <= 512, "four CTAs' tensor memory per SM");
struct ApplyParams {
  CUtensorMap tout;   // out as [N][H][64] bf16, box 64 channels x 1 head x 64 tokens, 128-byte swizzle
  CUtensorMap tq;     // Q as the state kernel's K and V (StateParams), when a map describes it
  LinearArgs a;
  int head_outer;
};

__device__ __forceinline__ void l_stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}
__device__ __forceinline__ uint32_t l_pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// D = f(Q) [S' | z] of one 64-token block: A = f(Q) (K-major, 64 tokens x 64
// channels), B = the [72][64] operand (K-major), N = 72, four K = 16 steps 32
// bytes apart; one elected lane issues and commits to `bar`.
__device__ __forceinline__ void apply_mma_elect(uint32_t d, uint64_t a, uint64_t b, uint64_t* bar) {
  constexpr uint32_t ID = tc::idesc(false, NB, false);
  asm volatile(
      "{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, 0, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %9, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %9, p1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%10];\n}\n"
      ::"r"(d), "l"(a), "l"(b), "l"(a + 2), "l"(b + 2), "l"(a + 4), "l"(b + 4), "l"(a + 6), "l"(b + 6), "r"(ID),
      "r"(tc::saddr(bar))
      : "memory");
}

static_assert(4 * (sizeof(ApplySmem) + 1024 + 1024) <= 228 * 1024, "four CTAs of the apply kernel per SM");

// f(Q) of block i over its own Q rows in ring stage `stage` (each thread reads and rewrites
// only the 32 bytes it copied), made visible to the tensor cores.
__device__ __forceinline__ void apply_prologue(const LinearArgs& a, unsigned char* stage, uint32_t oa, uint32_t ob,
                                               int tok, int half, int sub, int jb, bool valid) {
  const Geo& g = a.g;
  float xa[8], xb[8];
  read_q4(stage, oa, ob, xa, xb);
  bool sp;
  int row, col;
  view_pos(g, wrap_L(g, jb + tok), sp, row, col);
  features_lin<false>(xa, xb, half, sub, sp, row, col, a.rope_g, a.maxpos, a.eps, valid);
  store_q4(stage, oa, ob, xa, xb);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <bool TMA_IN>
__global__ void __launch_bounds__(LQ_THREADS, 4) linear_apply_q4_kernel(const __grid_constant__ ApplyParams prm) {
  // Software pipeline over the chunk's 64-token blocks, one barrier per block: while the
  // tensor cores compute block i's f(Q) [S' | z], the threads run block i + 1's prologue;
  // then block i's epilogue reads the accumulators, stages the bf16 rows by stmatrix in
  // output buffer i % 2, and one thread stores them by a bulk tensor copy (rows past the
  // tensor's last token are not written; chunks start on multiples of 64 tokens, so only
  // the last chunk has such rows) and issues block i + 1's MMAs.
  extern __shared__ unsigned char apply_smem_raw[];
  ApplySmem& sm = *reinterpret_cast<ApplySmem*>(align1024(apply_smem_raw));
  const LinearArgs& a = prm.a;
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x;   // grid (head, chunk), as in the state kernel
  const long long n0 = (long long)blockIdx.y * a.chunk_tokens;
  const long long n1 = min((long long)g.N, n0 + a.chunk_tokens);
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.q) + (long long)h * a.hs;
  const __nv_bfloat16* sb = static_cast<const __nv_bfloat16*>(a.state_b) + (size_t)h * NB * 64;
  const int tok = token_of(tid), half = (tid >> 1) & 1, sub = tid & 1;
  const int nblk = (int)((n1 - n0 + 63) / 64);
  const int left = (int)(n1 - n0) - tok;   // block i holds this thread's token iff 64 i < left
  const uint32_t oa = lswz(tok, 4 * half + sub), ob = lswz(tok, 4 * half + sub + 2);
  const uint32_t qst = lsmem(sm.q[0]), ost = lsmem(sm.out[0]);
  RowFetch fq(Q, n0, a.ts, tok, half, sub);
  int loaded = 0, seen = 0;   // blocks whose copies went out / whose landing this thread saw
  // block f (= loaded) into ring stage `stage` (bulk tensor copy armed by one thread, or 16-byte copies)
  auto load = [&](int f, int stage) {
    if constexpr (TMA_IN) {
      if (tid == 0) {
        const int n = (int)(n0 + 64LL * f);
        tc::mbar_expect_tx(&sm.full[stage], 64 * 128);
        l_tma_3d(qst + stage * 8192, &prm.tq, prm.head_outer ? n : h, prm.head_outer ? h : n, &sm.full[stage]);
      }
    } else {
      fq.fetch(qst + stage * 8192, oa, ob, 64 * f < left);
    }
    loaded = f + 1;
  };
  // block f's copies are complete for this thread (false: the wait ran out)
  auto landed = [&](int f) -> bool {
    if constexpr (TMA_IN) {
      if (!lin_wait(&sm.full[f % LA_STAGES], (f / LA_STAGES) & 1)) return false;
    } else {
      asm volatile("cp.async.wait_group %0;\n" ::"n"(LA_STAGES - 2));
    }
    seen = f + 1;
    return true;
  };
  if constexpr (!TMA_IN) {
    for (int i = 0; i < LA_STAGES - 1; ++i) {
      if (i < nblk) load(i, i);
      asm volatile("cp.async.commit_group;\n" ::);
    }
  }
  for (int i = tid; i < NB * 8; i += LQ_THREADS) {
    const int r = i >> 3, c = i & 7;
    *reinterpret_cast<uint4*>(sm.b + lswz(r, c)) = *reinterpret_cast<const uint4*>(sb + r * 64 + c * 8);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // B is read by the tensor cores
  if (tid == 0) {
    tc::mbar_init(&sm.mma_bar, 1);
    for (int i = 0; i < LA_STAGES; ++i) tc::mbar_init(&sm.full[i], 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(lsmem(&sm.tmem_base)),
                 "r"(APPLY_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // epilogue: warp w reads accumulator rows 16 (w % 4) .. + 15 (its TMEM lane quarter; 16x256b
  // shape: rows g4 and g4 + 8, columns 2 q4 and 2 q4 + 1 of each 8), columns 32 (w / 4) .. + 31
  // and the z column 64
  const int quarter = warp & 3, cg = warp >> 2, q4 = lane & 3;
  float bias[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = 32 * cg + 8 * j + 2 * q4;
    bias[2 * j] = a.b ? a.b[h * 64 + c] : 0.f;
    bias[2 * j + 1] = a.b ? a.b[h * 64 + c + 1] : 0.f;
  }
  // stmatrix row addresses in output buffer 0: lane 8 k + r gives row r of matrix k, matrices
  // (rows 0-7, n-block 2x), (rows 8-15, 2x), (rows 0-7, 2x + 1), (rows 8-15, 2x + 1) of store x
  const uint32_t o_st0 = ost + lswz(quarter * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), 4 * cg + (lane >> 4));
  const uint32_t o_st1 = ost + lswz(quarter * 16 + ((lane >> 3) & 1) * 8 + (lane & 7), 4 * cg + 2 + (lane >> 4));
  int jb = (int)(n0 % g.L);   // view position of the first token of the next block to prepare
  if constexpr (TMA_IN) {
    __syncthreads();   // the barriers are initialised: the first blocks go out
    for (int i = 0; i < LA_STAGES - 1; ++i)
      if (i < nblk) load(i, i);
  }
  if (nblk > 0) {
    if (!landed(0)) sm.abort = 1;
    apply_prologue(a, sm.q[0], oa, ob, tok, half, sub, jb, 0 < left);
    jb = wrap_L(g, jb + 64);
  }
  tc::fence_before();
  __syncthreads();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
  const uint64_t d_q0 = tc::desc_k(qst), d_b = tc::desc_k(lsmem(sm.b));
  if (warp == 0 && nblk > 0 && !sm.abort) {
    tc::fence_after();
    apply_mma_elect(tmem, d_q0, d_b, &sm.mma_bar);
  }
  int late = -1;   // thread 0: the block whose MMAs were not seen complete (abort)
  int st = 0, fst = LA_STAGES - 1;   // ring stages of block i and of block i - 1 (refilled now)
  for (int i = 0; i < nblk; ++i) {
    const int nst = ring_next(st, LA_STAGES);
    if (sm.abort) break;   // (read after the last barrier: the same in every thread)
    {   // block i + LA_STAGES - 1 into the stage of block i - 1 (its MMAs were seen complete
        // before the last barrier)
      const int f = i + LA_STAGES - 1;
      if (f < nblk) load(f, fst);
      if constexpr (!TMA_IN) asm volatile("cp.async.commit_group;\n" ::);
    }
    if (i + 1 < nblk) {   // block i + 1's copies (16-byte copies: the oldest but LA_STAGES - 2 groups)
      if (!landed(i + 1)) sm.abort = 1;
      apply_prologue(a, sm.q[nst], oa, ob, tok, half, sub, jb, 64 * (i + 1) < left);
      jb = wrap_L(g, jb + 64);
    }
    if (!lin_wait(&sm.mma_bar, i & 1)) {
      sm.abort = 1;
      if (tid == 0) late = i;
    }
    tc::fence_after();
    if (!sm.abort) {
      float r[16], z[4];
      tc::tmem_ld32(trow + 32 * cg, r);
      tc::tmem_ld8(trow + 64, z);
      // z = column 64 sits in z[0] (row g4) / z[2] (row g4 + 8) of the quad's first lane
      const float il0 = __fdividef(1.0f, __shfl_sync(0xffffffffu, z[0], lane & ~3));
      const float il1 = __fdividef(1.0f, __shfl_sync(0xffffffffu, z[2], lane & ~3));
      uint32_t w[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[j][0] = l_pack_bf16(fmaf(r[4 * j], il0, bias[2 * j]), fmaf(r[4 * j + 1], il0, bias[2 * j + 1]));
        w[j][1] = l_pack_bf16(fmaf(r[4 * j + 2], il1, bias[2 * j]), fmaf(r[4 * j + 3], il1, bias[2 * j + 1]));
      }
      const uint32_t ob_off = (i & 1) * 8192;
      l_stsm_x4(o_st0 + ob_off, w[0][0], w[0][1], w[1][0], w[1][1]);
      l_stsm_x4(o_st1 + ob_off, w[2][0], w[2][1], w[3][0], w[3][1]);
    }
    // the generic-proxy writes (output rows, block i + 1's f(Q)) become visible to the bulk
    // copy and the tensor cores; the TMEM reads are done before block i + 1's MMAs; block
    // i - 1's output copy has read its buffer before block i + 1's epilogue rewrites it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc::fence_before();
    if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
    __syncthreads();
    if (sm.abort) break;
    if (tid == 0) {
      asm volatile(
          "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];\n"
          "cp.async.bulk.commit_group;\n" ::"l"(&prm.tout), "r"(0), "r"(h), "r"((int)(n0 + 64LL * i)),
          "r"(ost + (i & 1) * 8192)
          : "memory");
    }
    if (warp == 0 && i + 1 < nblk) {
      tc::fence_after();
      apply_mma_elect(tmem, d_q0 + nst * 512, d_b, &sm.mma_bar);
    }
    st = nst;
    fst = ring_next(fst, LA_STAGES);
  }
  if constexpr (TMA_IN) {
    // after an abort, bulk copies that went out but were not waited for land first (bounded again)
    if (tid == 0 && sm.abort)
      for (int f = seen; f < loaded; ++f) lin_wait(&sm.full[f % LA_STAGES], (f / LA_STAGES) & 1);
  } else {
    asm volatile("cp.async.wait_group 0;\n" ::);
  }
  if (tid == 0) {
    asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
    if (late >= 0) lin_wait(&sm.mma_bar, late & 1);   // after an abort the late MMAs land first (bounded again)
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(APPLY_TMEM_COLS));
}

// --------------------------------------------------------------------------
// fp32 state
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) linear_state_simt_kernel(const __grid_constant__ LinearArgs a) {
  __shared__ float phi_s[64][65];
  __shared__ float v_s[64][64];
  const Geo& g = a.g;
  const int tid = threadIdx.x;
  const int h = blockIdx.y;
  const long long n0 = (long long)blockIdx.x * a.chunk_tokens;
  const long long n1 = min((long long)g.N, n0 + a.chunk_tokens);
  const float* K = static_cast<const float*>(a.k);
  const float* Vt = static_cast<const float*>(a.v);
  const int c = tid >> 2, jb = (tid & 3) * 16;
  float acc[16], zacc = 0.f;
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  for (long long nb = n0; nb < n1; nb += 64) {
    __syncthreads();
    if (tid < 64) {
      const long long n = nb + tid;
      float x[64];
      if (n < n1) {
        for (int e = 0; e < 64; ++e) x[e] = K[n * a.ts + (long long)h * a.hs + e];
        bool sp;
        int row, col;
        token_pos(g, n, sp, row, col);
        features_full(x, sp, row, col, a.rope, a.eps);
        for (int e = 0; e < 64; ++e) v_s[tid][e] = Vt[n * a.ts + (long long)h * a.hs + e];
      } else {
        for (int e = 0; e < 64; ++e) x[e] = 0.f, v_s[tid][e] = 0.f;
      }
      for (int e = 0; e < 64; ++e) phi_s[tid][e] = x[e];
    }
    __syncthreads();
    for (int tk = 0; tk < 64; ++tk) {
      const float p = phi_s[tk][c];
      for (int j = 0; j < 16; ++j) acc[j] = fmaf(p, v_s[tk][jb + j], acc[j]);
      zacc += p;
    }
  }
  float* part = a.part + ((size_t)blockIdx.x * g.H + h) * 64 * 65;
  for (int j = 0; j < 16; ++j) part[c * 65 + jb + j] = acc[j];
  if ((tid & 3) == 0) part[c * 65 + 64] = zacc;
}

// --------------------------------------------------------------------------
// 2. reduce + fold A: state[h][c][i] = sum_j S[c][j] A[i][j]; state[h][c][64] = z[c]
// --------------------------------------------------------------------------
// CTA = (head, 8 channel rows), 4 x 130 threads. The CTA's rows are 130
// 16-byte columns of every chunk partial; thread (slice, j) sums column j over
// the chunks ch = slice (mod 4), several copies in flight, and the four slice
// sums add in a fixed order (deterministic). Then the rows fold A in.
constexpr int RED_ROWS = 8;
constexpr int RED_VEC = RED_ROWS * 65 / 4;   // 130 16-byte columns
constexpr int RED_SLICES = 4;
constexpr int RED_THREADS = RED_VEC * RED_SLICES;
static_assert(RED_ROWS * 65 % 4 == 0, "whole 16-byte columns");
__global__ void __launch_bounds__(RED_THREADS) linear_reduce_kernel(const __grid_constant__ LinearArgs a, int want_bf16) {
  __shared__ float4 P[RED_SLICES][RED_VEC];
  __shared__ float S[RED_ROWS][65];
  __shared__ float As[64][65];
  const int h = blockIdx.x, c0 = blockIdx.y * RED_ROWS, tid = threadIdx.x;
  const Geo& g = a.g;
  {
    const int sl = tid / RED_VEC, j = tid - sl * RED_VEC;
    // rows c0.. of head h start 8 x 65 x 4 = 2,080 bytes apart: 16-byte aligned
    const float4* p = reinterpret_cast<const float4*>(a.part + ((size_t)h * 64 + c0) * 65) + j;
    const size_t cstride = (size_t)g.H * 64 * 65 / 4;   // 16-byte columns per chunk partial
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int ch = sl; ch < a.chunks; ch += RED_SLICES) {
      const float4 v = __ldg(p + (size_t)ch * cstride);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    P[sl][j] = s;
  }
  for (int e = tid; e < 64 * 64; e += RED_THREADS) {
    const int i = e / 64, j = e % 64;
    As[i][j] = a.A ? a.A[(size_t)h * 64 * 64 + e] : (i == j ? 1.f : 0.f);
  }
  __syncthreads();
  {
    const float* q = reinterpret_cast<const float*>(&P[0][0]);
    constexpr int E = RED_ROWS * 65;
    for (int e = tid; e < E; e += RED_THREADS) S[e / 65][e % 65] = (q[e] + q[E + e]) + (q[2 * E + e] + q[3 * E + e]);
  }
  __syncthreads();
  float* st = a.state + (size_t)h * 64 * 65;
  __nv_bfloat16* sb = want_bf16 ? static_cast<__nv_bfloat16*>(a.state_b) + (size_t)h * NB * 64 : nullptr;
  for (int e = tid; e < RED_ROWS * NB; e += RED_THREADS) {
    const int r = e / NB, i = e % NB, c = c0 + r;  // channel c, output column i
    float val = 0.f;
    if (i < 64) {
      for (int jj = 0; jj < 64; ++jj) val = fmaf(S[r][jj], As[i][jj], val);
    } else if (i == 64) {
      val = S[r][64];
    }
    if (i <= 64) st[c * 65 + i] = val;
    if (sb) sb[(size_t)i * 64 + c] = __float2bfloat16_rn(val);  // B operand stored [n][k]
  }
}

// fp32 apply: one thread per token
__global__ void __launch_bounds__(128) linear_apply_simt_kernel(const __grid_constant__ LinearArgs a) {
  __shared__ float st[64][65];
  const Geo& g = a.g;
  const int h = blockIdx.y;
  for (int e = threadIdx.x; e < 64 * 65; e += blockDim.x) st[e / 65][e % 65] = a.state[(size_t)h * 64 * 65 + e];
  __syncthreads();
  const long long n = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= g.N) return;
  const float* Q = static_cast<const float*>(a.q);
  float x[64];
  for (int e = 0; e < 64; ++e) x[e] = Q[n * a.ts + (long long)h * a.hs + e];
  bool sp;
  int row, col;
  token_pos(g, n, sp, row, col);
  features_full(x, sp, row, col, a.rope, a.eps);
  float den = 0.f;
  for (int c = 0; c < 64; ++c) den = fmaf(x[c], st[c][64], den);
  float* dst = static_cast<float*>(a.out) + (n * g.H + h) * D;
  for (int i = 0; i < 64; ++i) {
    float num = 0.f;
    for (int c = 0; c < 64; ++c) num = fmaf(x[c], st[c][i], num);
    dst[i] = num / den + (a.b ? a.b[h * 64 + i] : 0.f);
  }
}

// --------------------------------------------------------------------------
int linear_chunks(const Geo& g, int* chunk_tokens) {
  long long ct = 2048;
  long long chunks = (g.N + ct - 1) / ct;
  if (chunks > 256) {
    chunks = 256;
    ct = ((g.N + chunks - 1) / chunks + 63) / 64 * 64;
    chunks = (g.N + ct - 1) / ct;
  }
  if (chunks < 1) chunks = 1;
  *chunk_tokens = (int)ct;
  return (int)chunks;
}

// 3D bf16 map over out = [N][H][64] (contiguous), box 64 channels x 1 head x 64 tokens, 128-byte swizzle.
static bool make_out_map(CUtensorMap* m, void* out, const Geo& g) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  cuuint64_t dims[3] = {64, (cuuint64_t)g.H, (cuuint64_t)g.N};
  cuuint64_t strides[2] = {128, (cuuint64_t)g.H * 128};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// K or V ([N, H, 64] bf16 strided by ts, hs elements) as the state kernel's 3D map (see StateParams)
static bool make_in_map(CUtensorMap* m, const void* base, const Geo& g, long long ts, long long hs, int* head_outer) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  const cuuint64_t tsb = (cuuint64_t)ts * 2, hsb = g.H > 1 ? (cuuint64_t)hs * 2 : 128;
  if (tsb == 0 || hsb == 0 || tsb >= (1ull << 40) || hsb >= (1ull << 40)) return false;
  *head_outer = hsb > tsb ? 1 : 0;
  cuuint64_t dims[3] = {64, (cuuint64_t)(*head_outer ? g.N : g.H), (cuuint64_t)(*head_outer ? g.H : g.N)};
  cuuint64_t strides[2] = {*head_outer ? tsb : hsb, *head_outer ? hsb : tsb};
  cuuint32_t box[3] = {64, (cuuint32_t)(*head_outer ? 64 : 1), (cuuint32_t)(*head_outer ? 1 : 64)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <>
int launch_linear<__nv_bfloat16>(const LinearArgs& a, cudaStream_t st) {
  if (a.g.N == 0) return ZEBRA_OK;
  // the apply kernel's output copies cover whole 64-token blocks up to the tensor's end,
  // so only the last chunk may end inside a block
  if (a.chunk_tokens % 64) {
    set_error("linear stage: token chunks must be multiples of 64 tokens");
    return ZEBRA_ERR_UNSUPPORTED;
  }
  ApplyParams prm;
  prm.a = a;
  const bool tma_q = make_in_map(&prm.tq, a.q, a.g, a.ts, a.hs, &prm.head_outer);
  if (!make_out_map(&prm.tout, a.out, a.g)) {
    set_error("cuTensorMapEncodeTiled failed (linear output)");
    return ZEBRA_ERR_CUDA;
  }
  {
    StateParams sp;
    sp.a = a;
    int ho_k = 0, ho_v = 0;
    const bool tma_in = make_in_map(&sp.tk, a.k, a.g, a.ts, a.hs, &ho_k) &&
                        make_in_map(&sp.tv, a.v, a.g, a.ts, a.hs, &ho_v) && ho_k == ho_v;
    sp.head_outer = ho_k;
    ProfScope prof("linear_state", st);
    const int smem = (int)sizeof(StateSmem) + 1024;   // + alignment of the base to 1024 bytes
    auto kern = tma_in ? linear_state_q4_kernel<true> : linear_state_q4_kernel<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    kern<<<dim3(a.g.H, a.chunks), LQ_THREADS, smem, st>>>(sp);
  }
  count_launch();
  if (int rc = check_launch("linear_state_q4_kernel")) return rc;
  {
    ProfScope prof("linear_reduce", st);
    linear_reduce_kernel<<<dim3(a.g.H, 64 / RED_ROWS), RED_THREADS, 0, st>>>(a, 1);
  }
  count_launch();
  if (int rc = check_launch("linear_reduce_kernel")) return rc;
  {
    ProfScope prof("linear_apply", st);
    const int smem = (int)sizeof(ApplySmem) + 1024;   // + alignment of the base to 1024 bytes
    auto kern = tma_q ? linear_apply_q4_kernel<true> : linear_apply_q4_kernel<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    kern<<<dim3(a.g.H, a.chunks), LQ_THREADS, smem, st>>>(prm);
  }
  count_launch();
  return check_launch("linear_apply_q4_kernel");
}

template <>
int launch_linear<float>(const LinearArgs& a, cudaStream_t st) {
  if (a.g.N == 0) return ZEBRA_OK;
  {
    ProfScope prof("linear_state_simt", st);
    linear_state_simt_kernel<<<dim3(a.chunks, a.g.H), 256, 0, st>>>(a);
  }
  count_launch();
  if (int rc = check_launch("linear_state_simt_kernel")) return rc;
  {
    ProfScope prof("linear_reduce", st);
    linear_reduce_kernel<<<dim3(a.g.H, 64 / RED_ROWS), RED_THREADS, 0, st>>>(a, 0);
  }
  count_launch();
  if (int rc = check_launch("linear_reduce_kernel")) return rc;
  {
    ProfScope prof("linear_apply_simt", st);
    linear_apply_simt_kernel<<<dim3((unsigned)((a.g.N + 127) / 128), a.g.H), 128, 0, st>>>(a);
  }
  count_launch();
  return check_launch("linear_apply_simt_kernel");
}

}  // namespace zebra
