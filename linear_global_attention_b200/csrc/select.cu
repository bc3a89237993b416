// Per-query-tile key-tile selector.
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
// section "Linear-centered stages plus tile-sparse stages": the selector of a
// sparse stage retains a key-tile fraction of 1 - y for every query tile.
// This library scores key tile u for query tile t by the unscaled dot of their
// mean-pooled query and key (fp32), keeps the top k, and breaks equal scores
// toward the lower tile index.
//
// Per group of heads:
//  1. the scores S[h][t][u] = qm[h][t] . km[h][u] for all t, u, written to scratch:
//     scores_split_kernel splits the fp32 means into bf16 parts and one bf16
//     tensor-core GEMM (cuBLASLt, K = 6 x 64, fp32 accumulate, no split-K) sums the
//     part products to fp32 accuracy; scores_kernel, a 128x128-tile fp32 GEMM
//     with a fixed-order fma chain per score, is the CUDA-core alternative.
//  2. select_kernel: one CTA per row (h, t) copies the row into shared memory
//     (16-byte asynchronous copies, all in flight at once) and turns it into
//     order-preserving 32-bit keys, finds the k-th largest key from a 2,048-bin
//     histogram over the row's value range (a non-decreasing bin map; the bin
//     that holds the k-th key is found by a suffix scan; up to 256 of its keys
//     are ranked in one pass, up to 1,024 sorted; rows with a more crowded bin
//     take four 8-bit radix passes instead), then emits the bitmask: keys above
//     the threshold, plus the lowest-index keys equal to it (warp ballots per
//     mask word, a scan over warps when only some equal keys are kept).
//     It also flags near-ties: the k-th and (k+1)-th scores within a relative
//     gap of 1e-5.
#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"

namespace zebra {

// CTA = a 128 x 128 tile of S (query tiles t0.., key tiles u0..) of one head;
// the 64-channel means are staged channel-major in shared memory and every
// thread accumulates an 8 x 8 block with a fixed-order fma chain over the
// channels: rows 4 ty + i and 64 + 4 ty + i, columns 4 tx + j and 64 + 4 tx + j
// (i, j < 4), so each channel step reads four 16-byte vectors and each output
// row segment is stored as 16-byte vectors.
constexpr int SC_TILE = 128;
constexpr int SC_KC = 32;   // channels staged per step
__global__ void __launch_bounds__(256) scores_kernel(SelectArgs a) {
  __shared__ float sq[SC_KC][SC_TILE + 4];
  __shared__ float sk[SC_KC][SC_TILE + 4];
  const int T = a.g.T;
  const int hh = blockIdx.z;
  const int h = a.h0 + hh;
  const int t0 = blockIdx.y * SC_TILE, u0 = blockIdx.x * SC_TILE;
  const float* qm = a.qm + (size_t)h * T * D;
  const float* km = a.km + (size_t)h * T * D;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int c0 = 0; c0 < D; c0 += SC_KC) {
    __syncthreads();   // the previous channel block is consumed
    for (int i = threadIdx.x; i < SC_TILE * (SC_KC / 4); i += 256) {
      const int r = i / (SC_KC / 4), c4 = (i % (SC_KC / 4)) * 4;
      float4 q = make_float4(0, 0, 0, 0), k = q;
      if (t0 + r < T) q = *reinterpret_cast<const float4*>(qm + (size_t)(t0 + r) * D + c0 + c4);
      if (u0 + r < T) k = *reinterpret_cast<const float4*>(km + (size_t)(u0 + r) * D + c0 + c4);
      sq[c4][r] = q.x; sq[c4 + 1][r] = q.y; sq[c4 + 2][r] = q.z; sq[c4 + 3][r] = q.w;
      sk[c4][r] = k.x; sk[c4 + 1][r] = k.y; sk[c4 + 2][r] = k.z; sk[c4 + 3][r] = k.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < SC_KC; ++c) {
      float qv[8], kv[8];
      *reinterpret_cast<float4*>(qv) = *reinterpret_cast<const float4*>(&sq[c][4 * ty]);
      *reinterpret_cast<float4*>(qv + 4) = *reinterpret_cast<const float4*>(&sq[c][64 + 4 * ty]);
      *reinterpret_cast<float4*>(kv) = *reinterpret_cast<const float4*>(&sk[c][4 * tx]);
      *reinterpret_cast<float4*>(kv + 4) = *reinterpret_cast<const float4*>(&sk[c][64 + 4 * tx]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }
  }
  float* out = a.scores + (size_t)hh * T * a.Tld;
  // Tld is a multiple of 4, so every 4-column group starts on a 16-byte boundary
  // and lies wholly inside the row (columns T .. Tld - 1 are padding nobody reads)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + 4 * ty + (i & 3) + (i >> 2) * 64;
    if (t >= T) continue;
#pragma unroll
    for (int jh = 0; jh < 2; ++jh) {
      const int u = u0 + 4 * tx + jh * 64;
      if (u < a.Tld)
        *reinterpret_cast<float4*>(out + (size_t)t * a.Tld + u) =
            make_float4(acc[i][4 * jh], acc[i][4 * jh + 1], acc[i][4 * jh + 2], acc[i][4 * jh + 3]);
    }
  }
}

__device__ __forceinline__ uint32_t order_key(float s) {
  s = s + 0.0f;  // -0 -> +0: equal scores must map to equal keys
  const uint32_t f = __float_as_uint(s);
  return (f & 0x80000000u) ? ~f : (f | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

constexpr int SEL_THREADS = 512;
constexpr int HCOPIES = 8;
constexpr int HSTRIDE = 257;
constexpr int VBINS = 2048;      // bins of the value histogram (4 per thread)
constexpr int CAND_MAX = 1024;   // candidates of the threshold bin sorted exactly
constexpr int RANK_MAX = 256;    // up to this many candidates: ranks by one pass instead of a sort
constexpr int HIST_WORDS = HCOPIES * HSTRIDE > VBINS ? HCOPIES * HSTRIDE : VBINS;

__global__ void __launch_bounds__(SEL_THREADS) select_kernel(SelectArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[HIST_WORDS];
  __shared__ uint32_t cand[CAND_MAX];
  __shared__ uint32_t s_bin, s_need, s_eqtotal, s_ncand, s_thr, s_gt, s_eqn;
  __shared__ uint32_t s_wsum[SEL_THREADS / 32];
  __shared__ uint32_t s_max[SEL_THREADS / 32];
  __shared__ float s_vmin[SEL_THREADS / 32], s_vmax[SEL_THREADS / 32];
  const int T = a.g.T, W = a.g.W;
  const int t = blockIdx.x, hh = blockIdx.y, h = a.h0 + hh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* mrow = a.mask + ((size_t)h * T + t) * W;
  if (a.keep >= T) {
    for (int w = tid; w < W; w += SEL_THREADS) {
      const int rem = T - w * 32;
      mrow[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
    }
    if (a.near_tie && tid == 0) a.near_tie[(size_t)h * T + t] = 0;
    return;
  }
  // The row (Tld floats, a multiple of 4 starting on a 16-byte boundary) comes in
  // as 16-byte asynchronous copies, all in flight at once, and is then turned
  // into order keys in place.
  const float* srow = a.scores + ((size_t)hh * T + t) * a.Tld;
  for (int c = tid; c < (a.Tld >> 2); c += SEL_THREADS)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(keys + 4 * c))),
                 "l"(srow + 4 * c));
  asm volatile("cp.async.commit_group;\n" ::);
  asm volatile("cp.async.wait_group 0;\n" ::);
  __syncthreads();
  float vmin = INFINITY, vmax = -INFINITY;
  for (int i = tid; i < T; i += SEL_THREADS) {
    const float v = __uint_as_float(keys[i]);
    keys[i] = order_key(v);
    vmin = fminf(vmin, v);
    vmax = fmaxf(vmax, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if (lane == 0) {
    s_vmin[warp] = vmin;
    s_vmax[warp] = vmax;
  }
  for (int i = tid; i < VBINS; i += SEL_THREADS) hist[i] = 0;
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  vmin = s_vmin[0];
  vmax = s_vmax[0];
  for (int w = 1; w < SEL_THREADS / 32; ++w) {
    vmin = fminf(vmin, s_vmin[w]);
    vmax = fmaxf(vmax, s_vmax[w]);
  }
  // Value histogram: bin(v) = floor((v - vmin) * VBINS / (vmax - vmin)), a
  // non-decreasing function of v, so every key in a higher bin is larger than
  // every key in a lower one. The bin that holds the keep-th largest key is
  // found by a suffix scan; its keys are sorted exactly. Rows whose threshold
  // bin holds more than CAND_MAX keys (heavy ties) take the radix passes.
  const float span = vmax - vmin;
  const float scale = (float)VBINS / span;
  const bool binned = span > 0.f && isfinite(scale);
  uint32_t thr = 0, eq_take = 0, eq_total = 0;
  bool exact = false;
  if (binned) {
    for (int i = tid; i < T; i += SEL_THREADS) {
      const int bin = min(max((int)((key_value(keys[i]) - vmin) * scale), 0), VBINS - 1);
      atomicAdd(&hist[bin], 1u);
    }
    __syncthreads();
    // suffix scan over the bins: thread tid owns bins 4 (511 - tid) .. + 3, so
    // an inclusive prefix scan over tid runs from the top bin down
    const int b0 = 4 * (SEL_THREADS - 1 - tid);
    uint32_t c[4], sum = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c[e] = hist[b0 + 3 - e];
      sum += c[e];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    uint32_t base = 0;
    for (int w = 0; w < warp; ++w) base += s_wsum[w];
    incl += base;
    const uint32_t excl = incl - sum, need0 = (uint32_t)a.keep;
    if (excl < need0 && incl >= need0) {
      uint32_t cum = excl;
      int b = b0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (cum + c[e] >= need0) {
          b = b0 + 3 - e;
          break;
        }
        cum += c[e];
      }
      s_bin = (uint32_t)b;
      s_need = need0 - cum;
      s_eqtotal = hist[b];
    }
    __syncthreads();
    const int bsel = (int)s_bin;
    const uint32_t nbin = s_eqtotal, need_b = s_need;
    if (nbin <= (uint32_t)CAND_MAX) {
      for (int i = tid; i < T; i += SEL_THREADS) {
        const uint32_t k = keys[i];
        if (min(max((int)((key_value(k) - vmin) * scale), 0), VBINS - 1) == bsel) cand[atomicAdd(&s_ncand, 1u)] = k;
      }
      __syncthreads();
      uint32_t gt = 0, eq = 0;
      if (nbin <= (uint32_t)RANK_MAX) {
        // few candidates: candidate i's rank (larger keys, then equal keys at
        // lower slots) takes one pass over the candidates, read by all threads
        // at once; the candidate of rank need_b - 1 is the threshold
        if (tid < (int)nbin) {
          const uint32_t x = cand[tid];
          uint32_t n_gt = 0, n_eq = 0, n_eq_lo = 0;
          for (int j = 0; j < (int)nbin; ++j) {
            const uint32_t y = cand[j];
            n_gt += y > x ? 1u : 0u;
            n_eq += y == x ? 1u : 0u;
            n_eq_lo += (y == x && j < tid) ? 1u : 0u;
          }
          if (n_gt + n_eq_lo == need_b - 1) {
            s_thr = x;
            s_gt = n_gt;
            s_eqn = n_eq;
          }
        }
        __syncthreads();
        thr = s_thr;
        gt = s_gt;
        eq = s_eqn;
      } else {
        // the threshold bin's keys, sorted in descending order (bitonic, padded
        // with 0, below every order key of a finite score)
        int np = 1;
        while (np < (int)nbin) np <<= 1;
        for (int i = (int)nbin + tid; i < np; i += SEL_THREADS) cand[i] = 0u;
        __syncthreads();
        for (int kk = 2; kk <= np; kk <<= 1) {
          for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            for (int i = tid; i < np; i += SEL_THREADS) {
              const int l = i ^ jj;
              if (l > i) {
                const uint32_t x = cand[i], y = cand[l];
                const bool desc = (i & kk) == 0;
                if (desc ? x < y : x > y) {
                  cand[i] = y;
                  cand[l] = x;
                }
              }
            }
            __syncthreads();
          }
        }
        thr = cand[need_b - 1];
        // keys equal to the threshold: how many the bin holds, how many are taken
        for (int i = tid; i < (int)nbin; i += SEL_THREADS) {
          gt += cand[i] > thr ? 1u : 0u;
          eq += cand[i] == thr ? 1u : 0u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          gt += __shfl_xor_sync(0xffffffffu, gt, o);
          eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        __syncthreads();   // s_wsum / s_max are reused below
        if (lane == 0) {
          s_wsum[warp] = gt;
          s_max[warp] = eq;
        }
        __syncthreads();
        gt = 0;
        eq = 0;
        for (int w = 0; w < SEL_THREADS / 32; ++w) {
          gt += s_wsum[w];
          eq += s_max[w];
        }
      }
      eq_take = need_b - gt;
      eq_total = eq;
      exact = true;
    }
    __syncthreads();
  }
  if (!exact) {
    // radix passes over the whole row (all scores equal, or a crowded bin)
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)a.keep;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < HCOPIES * HSTRIDE; i += SEL_THREADS) hist[i] = 0;
      __syncthreads();
      uint32_t* hc = hist + (lane & (HCOPIES - 1)) * HSTRIDE;
      if (shift == 24) {
        // the top byte (sign and exponent bits) takes few distinct values: one
        // atomic per distinct bin per warp (the loop bound is uniform, so the
        // whole warp takes part in every match)
        for (int base = 0; base < T; base += SEL_THREADS) {
          const int i = base + tid;
          const uint32_t bin = i < T ? keys[i] >> 24 : 256u;
          const uint32_t peers = __match_any_sync(0xffffffffu, bin);
          if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hc[bin], (uint32_t)__popc(peers));
        }
      } else {
        for (int i = tid; i < T; i += SEL_THREADS) {
          const uint32_t k = keys[i];
          if ((k & pmask) == prefix) atomicAdd(&hc[(k >> shift) & 255u], 1u);
        }
      }
      __syncthreads();
      if (tid < 256) {
        uint32_t sum = 0;
#pragma unroll
        for (int c = 0; c < HCOPIES; ++c) sum += hist[c * HSTRIDE + tid];
        hist[tid] = sum;  // copy 0 slot tid: read by this thread only above
      }
      __syncthreads();
      if (warp == 0) {
        // the bin holding the need-th largest key: lane l owns bins 255 - 8 l
        // down to 248 - 8 l; an inclusive scan over the lanes (high bins first)
        // finds the lane where the running count reaches need
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[255 - 8 * lane - e];
          sum += c[e];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - sum;
        const unsigned hit = __ballot_sync(0xffffffffu, excl < need && incl >= need);
        if (lane == __ffs(hit) - 1) {
          uint32_t cum = excl;
          int b = 255 - 8 * lane - 7;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (cum + c[e] >= need) {
              b = 255 - 8 * lane - e;
              break;
            }
            cum += c[e];
          }
          s_bin = (uint32_t)b;
          s_need = need - cum;
          s_eqtotal = hist[b];
        }
      }
      __syncthreads();
      prefix |= s_bin << shift;
      pmask |= 255u << shift;
      need = s_need;
      __syncthreads();
    }
    thr = prefix;
    eq_take = need;
    eq_total = s_eqtotal;
  }
  // thr: the keep-th largest key; eq_take of the eq_total keys equal to it are
  // kept, lowest index first

  // mask words: warp w owns a contiguous run of words and reads them a word at a
  // time, lane j holding key 32 word + j (bank-conflict free); two ballots give
  // the word's "greater" and "equal" bits.
  constexpr int NWARP = SEL_THREADS / 32;
  const int wpw = (W + NWARP - 1) / NWARP;
  const int wa = min(W, warp * wpw), wb = min(W, wa + wpw);
  uint32_t before = 0;   // equal keys at lower indices than the current word
  if (eq_take < eq_total) {
    // only some equal keys are kept: the lowest-index ones, so each warp needs
    // the count of equal keys in the words of the warps before it
    uint32_t cnt = 0;
    for (int w = wa; w < wb; ++w) {
      const int i = w * 32 + lane;
      cnt += __popc(__ballot_sync(0xffffffffu, i < T && keys[i] == thr));
    }
    if (lane == 0) s_wsum[warp] = cnt;
    __syncthreads();
    for (int x = 0; x < warp; ++x) before += s_wsum[x];
  }
  for (int w = wa; w < wb; ++w) {
    const int i = w * 32 + lane;
    const uint32_t k = i < T ? keys[i] : 0u;
    const uint32_t gt = __ballot_sync(0xffffffffu, i < T && k > thr);
    uint32_t eqb = __ballot_sync(0xffffffffu, i < T && k == thr);
    const uint32_t ne = (uint32_t)__popc(eqb);
    // with every equal key kept (eq_take >= eq_total) the local count suffices:
    // it never exceeds the global one, so take == ne
    uint32_t take = before >= eq_take ? 0u : min(eq_take - before, ne);
    before += ne;
    uint32_t keepb = 0;
    if (take == ne) {
      keepb = eqb;
    } else {
      while (take--) {
        const uint32_t low = eqb & (~eqb + 1u);
        keepb |= low;
        eqb ^= low;
      }
    }
    if (lane == 0) mrow[w] = gt | keepb;
  }

  if (a.near_tie) {
    // (k+1)-th largest: equal to thr if more keys equal it than were taken,
    // otherwise the largest key below thr
    uint32_t below = 0;
    if (eq_total <= eq_take) {
      for (int i = tid; i < T; i += SEL_THREADS) {
        const uint32_t k = keys[i];
        if (k < thr && k > below) below = k;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) below = max(below, __shfl_xor_sync(0xffffffffu, below, o));
    if (lane == 0) s_max[warp] = below;
    __syncthreads();
    if (tid == 0) {
      uint32_t nxt = 0;
      for (int i = 0; i < SEL_THREADS / 32; ++i) nxt = max(nxt, s_max[i]);
      uint8_t flag;
      if (eq_total > eq_take) {
        flag = 1;
      } else {
        const double s_a = key_value(thr), s_b = key_value(nxt);
        const double den = fmax(fabs(s_a), fabs(s_b));
        const double gap = den > 0 ? fabs(s_a - s_b) / den : 0.0;
        flag = gap < 1e-5 ? 1 : 0;
      }
      a.near_tie[(size_t)h * T + t] = flag;
    }
  }
}

// Scores on the tensor cores. Each fp32 mean x is split into three bf16 parts,
// x = x0 + x1 + x2 up to 2^-24 relative (x0 = bf16(x), x1 = bf16(x - x0),
// x2 = bf16(x - x0 - x1); both subtractions are exact in fp32). The score
// q . k = sum over the part pairs of q_a . k_b; the six pairs with a + b <= 2
// leave out terms of relative size 2^-24 and below. Laid out as one bf16 GEMM
// with K = 6 x 64, Q'[t] = [q0 q0 q1 q0 q1 q2] and K'[u] = [k0 k1 k0 k2 k1 k0],
// with fp32 accumulation: the score error is that of an fp32 dot product,
// and equal key means give equal scores (every element sums its products in
// the same order).
__global__ void __launch_bounds__(128) scores_split_kernel(SelectArgs a) {
  const int T = a.g.T;
  const int t = blockIdx.x * 2 + (threadIdx.x >> 6), c = threadIdx.x & 63;
  const int hh = blockIdx.y, h = a.h0 + hh;
  if (t >= T) return;
  auto parts = [](float x, __nv_bfloat16& p0, __nv_bfloat16& p1, __nv_bfloat16& p2) {
    p0 = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(p0);
    p1 = __float2bfloat16_rn(r1);
    p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
  };
  __nv_bfloat16 q0, q1, q2, k0, k1, k2;
  parts(a.qm[((size_t)h * T + t) * D + c], q0, q1, q2);
  parts(a.km[((size_t)h * T + t) * D + c], k0, k1, k2);
  __nv_bfloat16* qs = static_cast<__nv_bfloat16*>(a.qsplit) + ((size_t)hh * T + t) * SPLIT_K + c;
  __nv_bfloat16* ks = static_cast<__nv_bfloat16*>(a.ksplit) + ((size_t)hh * T + t) * SPLIT_K + c;
  qs[0] = q0; qs[64] = q0; qs[128] = q1; qs[192] = q0; qs[256] = q1; qs[320] = q2;
  ks[0] = k0; ks[64] = k1; ks[128] = k0; ks[192] = k2; ks[256] = k1; ks[320] = k0;
}

#ifndef ZEBRA_SCORES_TC
#define ZEBRA_SCORES_TC 1
#endif

int launch_scores(const SelectArgs& a, cudaStream_t st) {
  const int T = a.g.T;
  if (T == 0 || a.keep >= T) return ZEBRA_OK;
  ProfScope prof("tile_scores", st);
  if (ZEBRA_SCORES_TC && a.qsplit) {
    scores_split_kernel<<<dim3((T + 1) / 2, a.hc), 128, 0, st>>>(a);
    count_launch();
    if (int rc = check_launch("scores_split_kernel")) return rc;
    return gemm_bf16_nt_f32(a.qsplit, a.ksplit, a.scores, T, T, SPLIT_K, a.Tld, a.hc, (long long)T * SPLIT_K,
                            (long long)T * SPLIT_K, (long long)T * a.Tld, a.gemm_ws, a.gemm_ws_bytes, st);
  }
  dim3 grid((T + SC_TILE - 1) / SC_TILE, (T + SC_TILE - 1) / SC_TILE, a.hc);
  scores_kernel<<<grid, 256, 0, st>>>(a);
  count_launch();
  return check_launch("scores_kernel");
}

int launch_select(const SelectArgs& a, cudaStream_t st) {
  const int T = a.g.T;
  if (T == 0) return ZEBRA_OK;
  const size_t smem = (size_t)a.Tld * sizeof(uint32_t);   // whole 16-byte chunks of the row
  cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SELECT_MAX_T * 4);
  dim3 grid(T, a.hc);
  ProfScope prof("tile_select", st);
  select_kernel<<<grid, SEL_THREADS, smem, st>>>(a);
  count_launch();
  return check_launch("select_kernel");
}

}  // namespace zebra
