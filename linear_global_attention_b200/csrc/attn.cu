// Tile-sparse softmax attention and dense special-token rows.
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
// section "Linear-centered stages plus tile-sparse stages": selected tiles keep
// full softmax interactions, omitted tiles are summarised as mean key/value
// landmarks, special-token keys stay visible, special-token query rows keep
// dense attention, and every patch query retains its own self key.
//
// One CTA handles one (query tile, head) and runs a single online softmax over
// a stream of 64-key blocks:
//   kind 0  a kept key tile (packed, rows >= n_u masked),
//   kind 1  64 landmark rows (mean K/V of tiles u..u+63), logit bias ln(n_u),
//           masked where u is kept, u is the own tile, or u >= T,
//   kind 2  64 special-token keys (rows >= NS masked),
// followed, when the own tile is not kept, by two per-row entries: the exact
// self key and the own-tile landmark over the other n_t - 1 tokens.
// All logits carry the 1/sqrt(d) scale; exponentials are base 2 with log2(e)
// folded into the scale and biases.
//
// bf16 patch rows run on the tcgen05 kernel (attn_tc.cuh, included below).
// fp32 path: one thread per query row, plain fp32 arithmetic (small inputs).
//
// Special-token query rows attend all N keys: split-KV over key-tile ranges,
// partial (max, sum, unnormalised output) per split, then a combine kernel. In
// bf16 they run on the tcgen05 kernel (attn_tc.cuh, mode 1); in fp32 on one
// thread per row.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace zebra {

// Visible (unmasked) logits evaluated: [0] patch rows of the sparse kernel,
// [1] special-token rows. Each costs 4*d FLOPs (QK^T and PV); one atomic per CTA.
__device__ unsigned long long g_logits[2];

void reset_logit_counters() {
  const unsigned long long z[2] = {0, 0};
  cudaMemcpyToSymbol(g_logits, z, sizeof(z));
}
void read_logit_counters(unsigned long long* out2) { cudaMemcpyFromSymbol(out2, g_logits, 2 * sizeof(unsigned long long)); }

// ---------------------------------------------------------------------------
// block stream
// ---------------------------------------------------------------------------
struct BlockIter {
  int phase;      // 0 kept tiles, 1 landmark blocks, 2 special blocks, 3 done
  int w;          // mask word (phase 0) / tile cursor (dense rows)
  uint32_t bits;
  uint32_t nxt;   // word w + 1, loaded one word ahead
  int lb, sb;
  int t_end;      // dense rows: end of the tile range
};

// word w of a selection row, with bits of tiles >= T cleared (a caller-supplied
// mask may carry stray bits there)
__device__ __forceinline__ uint32_t mask_word(const uint32_t* __restrict__ mrow, int w, int T) {
  const uint32_t m = __ldg(mrow + w);
  const int rem = T - w * 32;
  return rem >= 32 ? m : (m & ((1u << rem) - 1u));
}

// start the kept-tile walk of selection row `mrow`
__device__ __forceinline__ void iter_init(BlockIter& it, const uint32_t* __restrict__ mrow, const Geo& g) {
  it.bits = mask_word(mrow, 0, g.T);
  it.nxt = g.W > 1 ? mask_word(mrow, 1, g.T) : 0u;
}

// Landmarks of block lb (landmarks 64 lb .. 64 lb + 63) visible to query tile
// t: tiles below T, not selected, not t itself. Returns their bit set over the
// two mask words; `nvis` gets their count.
__device__ __forceinline__ uint32_t lmk_visible(const uint32_t* __restrict__ mrow, const Geo& g, int t, int lb,
                                                int& nvis) {
  uint32_t vis = 0;
  nvis = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int w = lb * 2 + k;
    if (w >= g.W) continue;
    uint32_t inr = 0xffffffffu;
    const int rem = g.T - w * 32;
    if (rem < 32) inr = (1u << rem) - 1u;
    uint32_t v = ~__ldg(mrow + w) & inr;
    if ((t >> 5) == w) v &= ~(1u << (t & 31));
    vis |= v;
    nvis += __popc(v);
  }
  return vis;
}

// MODE 0: the kept tiles of row `mrow`, then landmark blocks with at least one
// visible landmark, then special blocks. `it` starts from iter_init.
__device__ __forceinline__ bool next_block_sparse(BlockIter& it, const Geo& g, const uint32_t* __restrict__ mrow,
                                                  int t, bool has_lmk, int& kind, int& id, int& nv) {
  if (it.phase == 0) {
    while (it.bits == 0 && it.w + 1 < g.W) {
      ++it.w;
      it.bits = it.nxt;
      it.nxt = it.w + 1 < g.W ? mask_word(mrow, it.w + 1, g.T) : 0u;
    }
    if (it.bits != 0) {
      const int b = __ffs(it.bits) - 1;
      it.bits &= it.bits - 1;
      kind = 0;
      id = it.w * 32 + b;
      const TileShape ts = tile_shape(g, id);
      nv = ts.rows * ts.cols;
      return true;
    }
    it.phase = 1;
  }
  if (it.phase == 1) {
    if (has_lmk) {
      const int nlb = g.Tpad / 64;
      while (it.lb < nlb) {
        const int lb = it.lb++;
        int nvis;
        const uint32_t vis = lmk_visible(mrow, g, t, lb, nvis);
        if (vis) {
          kind = 1;
          id = lb;
          nv = nvis;
          return true;
        }
      }
    }
    it.phase = 2;
  }
  if (it.phase == 2) {
    if (it.sb < g.NSp / 64) {
      kind = 2;
      id = it.sb++;
      nv = min(64, g.NS - id * 64);
      return true;
    }
    it.phase = 3;
  }
  return false;
}

// MODE 1: tiles [w, t_end), then the special blocks when `with_special`.
__device__ __forceinline__ bool next_block_dense(BlockIter& it, const Geo& g, bool with_special, int& kind, int& id,
                                                 int& nv) {
  if (it.phase == 0) {
    if (it.w < it.t_end) {
      kind = 0;
      id = it.w++;
      const TileShape ts = tile_shape(g, id);
      nv = ts.rows * ts.cols;
      return true;
    }
    it.phase = 2;
  }
  if (it.phase == 2 && with_special && it.sb < g.NSp / 64) {
    kind = 2;
    id = it.sb++;
    nv = min(64, g.NS - id * 64);
    return true;
  }
  it.phase = 3;
  return false;
}

// bias (log2 units) of column j of a block; -inf = masked
__device__ __forceinline__ float block_bias(const AttnArgs& a, const uint32_t* __restrict__ mrow, int t, int kind,
                                            int id, int j) {
  const Geo& g = a.g;
  const float NEG = -INFINITY;
  if (kind == 0) {
    const TileShape s = tile_shape(g, id);
    return j < s.rows * s.cols ? 0.f : NEG;
  }
  if (kind == 1) {
    const int u = id * 64 + j;
    if (u >= g.T || u == t) return NEG;
    if ((__ldg(mrow + (u >> 5)) >> (u & 31)) & 1u) return NEG;
    return __ldg(a.lmk_bias + u);   // ln(n_u) log2(e), written by the pooling pass
  }
  return id * 64 + j < g.NS ? 0.f : NEG;
}

template <typename T>
__device__ __forceinline__ void block_src(const AttnArgs& a, int h, int kind, int id, const T*& k, const T*& v) {
  const Geo& g = a.g;
  if (kind == 0) {
    const size_t off = ((size_t)h * g.T + id) * TOK * D;
    k = static_cast<const T*>(a.Kp) + off;
    v = static_cast<const T*>(a.Vp) + off;
  } else if (kind == 1) {
    const size_t off = ((size_t)h * g.Tpad + (size_t)id * 64) * D;
    k = static_cast<const T*>(a.Kl) + off;
    v = static_cast<const T*>(a.Vl) + off;
  } else {
    const size_t off = ((size_t)h * g.NSp + (size_t)id * 64) * D;
    k = static_cast<const T*>(a.Ks) + off;
    v = static_cast<const T*>(a.Vs) + off;
  }
}

// ---------------------------------------------------------------------------
// mma.sync helpers (the attention-concentration diagnostic)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte offset of (row, 16-byte chunk) in a swizzled 64x64 bf16 tile
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------
// attention-concentration diagnostic (page section "Sensitive stages also
// concentrate their attention"): for each row of a sampled patch query tile,
// the dense softmax mass (scale 1/sqrt(d), all N keys) that falls on the
// tokens of the tile's selected key tiles and on the special-token keys.
// CTA = (sampled tile, head, key split), 4 warps x 16 query rows, mma.sync
// QK^T over 64-key blocks read straight from the strided K; per row a running
// maximum and three sums (all keys, selected tiles, special keys) in the same
// units; coverage_combine_kernel merges the splits in a fixed order.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) coverage_kernel(const __grid_constant__ CoverageArgs a) {
  __shared__ __align__(128) __nv_bfloat16 qs[64 * 64];
  __shared__ __align__(128) __nv_bfloat16 ks[2][64 * 64];
  __shared__ float bias[2][64];
  __shared__ int kind_sh[2];   // 0 unselected tile, 1 selected tile, 2 special block
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
  const int t = a.tiles[i];
  const uint32_t* mrow = a.mask + ((size_t)h * g.T + t) * g.W;
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.q) + (long long)h * a.hs;
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.k) + (long long)h * a.hs;
  const TileShape qt = tile_shape(g, t);
  const int n_t = qt.rows * qt.cols;
  for (int e = tid; e < 512; e += 128) {
    const int r = e >> 3, c = e & 7;
    if (r < n_t) cp_async16(smem_u32(qs) + swz(r, c), Q + tile_token(g, qt, r) * a.ts + c * 8);
    else store16_zero(reinterpret_cast<char*>(qs) + swz(r, c));
  }
  cp_async_commit();
  const int u0 = (int)((long long)g.T * sp / a.splits), u1 = (int)((long long)g.T * (sp + 1) / a.splits);
  const int nspec = sp == 0 ? g.NSp / 64 : 0;
  const int nblk = (u1 - u0) + nspec;
  // block b: key tile u0 + b, then the special blocks
  auto issue = [&](int b, int buf) {
    if (b < u1 - u0) {
      const int u = u0 + b;
      const TileShape ks_ = tile_shape(g, u);
      const int n_u = ks_.rows * ks_.cols;
      for (int e = tid; e < 512; e += 128) {
        const int r = e >> 3, c = e & 7;
        if (r < n_u) cp_async16(smem_u32(ks[buf]) + swz(r, c), K + tile_token(g, ks_, r) * a.ts + c * 8);
        else store16_zero(reinterpret_cast<char*>(ks[buf]) + swz(r, c));
      }
      if (tid < 64) bias[buf][tid] = tid < n_u ? 0.f : -INFINITY;
      if (tid == 0) kind_sh[buf] = (int)((__ldg(mrow + (u >> 5)) >> (u & 31)) & 1u);
    } else {
      const int sb = b - (u1 - u0);
      for (int e = tid; e < 512; e += 128) {
        const int r = e >> 3, c = e & 7, si = sb * 64 + r;
        if (si < g.NS) cp_async16(smem_u32(ks[buf]) + swz(r, c), K + special_token(g, si) * a.ts + c * 8);
        else store16_zero(reinterpret_cast<char*>(ks[buf]) + swz(r, c));
      }
      if (tid < 64) bias[buf][tid] = sb * 64 + tid < g.NS ? 0.f : -INFINITY;
      if (tid == 0) kind_sh[buf] = 2;
    }
  };
  if (nblk > 0) issue(0, 0);
  cp_async_commit();
  const float sc = LOG2E * 0.125f;
  const int g4 = lane >> 2, q4 = lane & 3;
  float m[2] = {-INFINITY, -INFINITY}, z[2] = {0.f, 0.f}, ssel[2] = {0.f, 0.f}, sspec[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  for (int b = 0; b < nblk; ++b) {
    const int buf = b & 1;
    if (b + 1 < nblk) issue(b + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (b == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int mi = lane >> 3, ri = lane & 7;
        ldsm_x4(smem_u32(qs) + swz(warp * 16 + (mi & 1) * 8 + ri, 2 * kk + (mi >> 1)), qf[kk][0], qf[kk][1],
                qf[kk][2], qf[kk][3]);
      }
    }
    float sv[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sv[j][0] = sv[j][1] = sv[j][2] = sv[j][3] = 0.f;
    const uint32_t kb = smem_u32(ks[buf]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int mi = lane >> 3, ri = lane & 7;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz(np * 16 + (mi >> 1) * 8 + ri, 2 * kk + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(sv[2 * np], qf[kk], b0, b1);
        mma_bf16(sv[2 * np + 1], qf[kk], b2, b3);
      }
    }
    const int kind = kind_sh[buf];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float& x = sv[j][2 * half + e];
          x = fmaf(x, sc, bias[buf][8 * j + 2 * q4 + e]);
          mx = fmaxf(mx, x);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(m[half], mx);
      const float base = mn == -INFINITY ? 0.f : mn;
      const float al = exp2f(m[half] - base);
      float ps = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) ps += exp2f(sv[j][2 * half] - base) + exp2f(sv[j][2 * half + 1] - base);
      m[half] = mn;
      z[half] = z[half] * al + ps;
      ssel[half] = ssel[half] * al + (kind == 1 ? ps : 0.f);
      sspec[half] = sspec[half] * al + (kind == 2 ? ps : 0.f);
    }
    __syncthreads();   // the buffer is reloaded by the next issue
  }
  cp_async_wait<0>();
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      z[half] += __shfl_xor_sync(0xffffffffu, z[half], o);
      ssel[half] += __shfl_xor_sync(0xffffffffu, ssel[half], o);
      sspec[half] += __shfl_xor_sync(0xffffffffu, sspec[half], o);
    }
    if (q4 == 0) {
      const int r = warp * 16 + g4 + 8 * half;
      a.part[(((size_t)i * g.H + h) * a.splits + sp) * 64 + r] = make_float4(m[half], z[half], ssel[half], sspec[half]);
    }
  }
}

// merge the splits of every (sampled tile, head, row): fixed order
__global__ void coverage_combine_kernel(const __grid_constant__ CoverageArgs a) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)a.n * a.g.H * 64) return;
  const int r = (int)(e & 63);
  const long long ih = e >> 6;   // i * H + h
  const int i = (int)(ih / a.g.H);
  const TileShape qt = tile_shape(a.g, a.tiles[i]);
  if (r >= qt.rows * qt.cols) {
    a.sel[e] = 0.f;
    a.spec[e] = 0.f;
    return;
  }
  const float4* p = a.part + ih * a.splits * 64 + r;
  float mstar = -INFINITY;
  for (int s = 0; s < a.splits; ++s) mstar = fmaxf(mstar, p[s * 64].x);
  float z = 0.f, ss = 0.f, sp = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float4 v = p[s * 64];
    if (v.x == -INFINITY) continue;
    const float w = exp2f(v.x - mstar);
    z += w * v.y;
    ss += w * v.z;
    sp += w * v.w;
  }
  a.sel[e] = ss / z;
  a.spec[e] = sp / z;
}

int coverage_splits(const Geo& g, int n) {
  long long s = (4LL * 148 + (long long)n * g.H - 1) / ((long long)n * g.H);
  if (s > 64) s = 64;
  if (s > g.T) s = g.T;
  return (int)(s < 1 ? 1 : s);
}

int launch_coverage(const CoverageArgs& a, cudaStream_t st) {
  {
    ProfScope prof("coverage", st);
    coverage_kernel<<<dim3(a.n, a.g.H, a.splits), 128, 0, st>>>(a);
  }
  count_launch();
  if (int rc = check_launch("coverage_kernel")) return rc;
  const long long threads = (long long)a.n * a.g.H * 64;
  {
    ProfScope prof("coverage_combine", st);
    coverage_combine_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(a);
  }
  count_launch();
  return check_launch("coverage_combine_kernel");
}

// ---------------------------------------------------------------------------
// fp32 path (one thread per query row)
// ---------------------------------------------------------------------------
struct SimtSmem {
  float k[64][64];
  float v[64][64];
  float bias[64];
};

template <int MODE>
__global__ void __launch_bounds__(64) attn_simt_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ SimtSmem sm;
  const Geo& g = a.g;
  const int r = threadIdx.x;
  const int h = blockIdx.y, t = blockIdx.x;
  const uint32_t* mrow = MODE == 0 ? a.mask + ((size_t)h * g.T + t) * g.W : nullptr;
  const float* qsrc = MODE == 0 ? static_cast<const float*>(a.Qp) + ((size_t)h * g.T + t) * TOK * D
                                : static_cast<const float*>(a.Qs) + ((size_t)h * g.NSp + (size_t)t * 64) * D;
  float q[64], acc[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    q[c] = qsrc[r * D + c];
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const float sc = LOG2E * 0.125f;
  BlockIter it{};
  bool with_special = true, own_kept = true;
  int n_t = 0;
  if (MODE == 0) {
    iter_init(it, mrow, g);
    own_kept = (__ldg(mrow + (t >> 5)) >> (t & 31)) & 1u;
    const TileShape s = tile_shape(g, t);
    n_t = s.rows * s.cols;
  } else {
    const int sp = blockIdx.z;
    it.w = (int)((long long)g.T * sp / a.splits);
    it.t_end = (int)((long long)g.T * (sp + 1) / a.splits);
    with_special = sp == 0;
  }
  int kind, id, nv;
  while (MODE == 0 ? next_block_sparse(it, g, mrow, t, true, kind, id, nv)
                   : next_block_dense(it, g, with_special, kind, id, nv)) {
    const float *ks, *vs;
    block_src<float>(a, h, kind, id, ks, vs);
    __syncthreads();
    for (int i = r; i < 64 * 64; i += 64) {
      sm.k[i / 64][i % 64] = ks[i];
      sm.v[i / 64][i % 64] = vs[i];
    }
    sm.bias[r] = block_bias(a, mrow, t, kind, id, r);
    __syncthreads();
    for (int j = 0; j < 64; ++j) {
      const float b = sm.bias[j];
      if (b == -INFINITY) continue;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) dot = fmaf(q[c], sm.k[j][c], dot);
      const float s = fmaf(dot, sc, b);
      const float mn = fmaxf(m, s);
      const float al = exp2f(m - mn), p = exp2f(s - mn);
      m = mn;
      l = l * al + p;
#pragma unroll
      for (int c = 0; c < 64; ++c) acc[c] = fmaf(acc[c], al, p * sm.v[j][c]);
    }
  }
  if (MODE == 0) {
    if (!own_kept) {
      const size_t tb = ((size_t)h * g.T + t) * TOK * D;
      const float* Kp = static_cast<const float*>(a.Kp) + tb + r * D;
      const float* Vp = static_cast<const float*>(a.Vp) + tb + r * D;
      const float* km = a.km + ((size_t)h * g.T + t) * D;
      const float* vm = a.vm + ((size_t)h * g.T + t) * D;
      float qk = 0.f, qm = 0.f;
      for (int c = 0; c < 64; ++c) {
        qk = fmaf(q[c], Kp[c], qk);
        qm = fmaf(q[c], km[c], qm);
      }
      const float nt = (float)n_t;
      const float s_self = qk * sc;
      const float s_lm = n_t > 1 ? (nt * qm - qk) / (nt - 1.f) * sc + a.ln_tab[n_t - 1] * LOG2E : -INFINITY;
      const float mn = fmaxf(m, fmaxf(s_self, s_lm));
      const float al = exp2f(m - mn), ps = exp2f(s_self - mn), pl = n_t > 1 ? exp2f(s_lm - mn) : 0.f;
      l = l * al + ps + pl;
      for (int c = 0; c < 64; ++c) {
        const float vl = n_t > 1 ? (nt * vm[c] - Vp[c]) / (nt - 1.f) : 0.f;
        acc[c] = acc[c] * al + ps * Vp[c] + pl * vl;
      }
    }
    if (r < n_t) {
      const TileShape s = tile_shape(g, t);
      float* dst = static_cast<float*>(a.out) + (tile_token(g, s, r) * g.H + h) * D;
      const float il = 1.0f / l;
      for (int c = 0; c < 64; ++c) dst[c] = acc[c] * il;
    }
  } else {
    const int sp = blockIdx.z;
    const size_t row = ((size_t)sp * g.H + h) * g.NSp + (size_t)t * 64 + r;
    for (int c = 0; c < 64; ++c) a.part_o[row * D + c] = acc[c];
    a.part_ml[row * 2] = m;
    a.part_ml[row * 2 + 1] = l;
  }
}

// ---------------------------------------------------------------------------
// split-KV combine of the special-token rows: one warp per (special query, head)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void special_combine_kernel(const __grid_constant__ AttnArgs a) {
  const Geo& g = a.g;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)g.NS * g.H) return;
  const int h = (int)(wid % g.H), i = (int)(wid / g.H);
  float mstar = -INFINITY;
  for (int s = 0; s < a.splits; ++s) mstar = fmaxf(mstar, a.part_ml[(((size_t)s * g.H + h) * g.NSp + i) * 2]);
  float l = 0.f, o0 = 0.f, o1 = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const size_t row = ((size_t)s * g.H + h) * g.NSp + i;
    const float ms = a.part_ml[row * 2];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - mstar);
    l += w * a.part_ml[row * 2 + 1];
    o0 += w * a.part_o[row * D + 2 * lane];
    o1 += w * a.part_o[row * D + 2 * lane + 1];
  }
  T* dst = static_cast<T*>(a.out) + (special_token(g, i) * g.H + h) * D + 2 * lane;
  dst[0] = Elem<T>::from_f(o0 / l);
  dst[1] = Elem<T>::from_f(o1 / l);
}

}  // namespace zebra

#include "attn_tc.cuh"

namespace zebra {

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <>
int launch_sparse_attn<__nv_bfloat16>(const AttnArgs& a, cudaStream_t st) {
  return launch_sparse_attn_tc(a, st);
}
template <>
int launch_sparse_attn<float>(const AttnArgs& a, cudaStream_t st) {
  if (a.g.T == 0) return ZEBRA_OK;
  ProfScope prof("attn_sparse_rows_f32", st);
  attn_simt_kernel<0><<<dim3(a.g.T, a.g.H), 64, 0, st>>>(a);
  count_launch();
  return check_launch("attn_simt_kernel<sparse>");
}

template <typename T>
int launch_special_rows(const AttnArgs& a, cudaStream_t st) {
  if (a.g.NS == 0) return ZEBRA_OK;
  if (sizeof(T) == 2) {
    if (int rc = launch_special_rows_tc(a, st)) return rc;
  } else {
    dim3 grid(a.g.NSp / 64, a.g.H, a.splits);
    {
      ProfScope prof("attn_special_rows_f32", st);
      attn_simt_kernel<1><<<grid, 64, 0, st>>>(a);
    }
    count_launch();
    if (int rc = check_launch("attn_simt_kernel<special rows>")) return rc;
  }
  const long long threads = (long long)a.g.NS * a.g.H * 32;
  ProfScope prof("special_combine", st);
  special_combine_kernel<T><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(a);
  count_launch();
  return check_launch("special_combine_kernel");
}

template int launch_special_rows<float>(const AttnArgs&, cudaStream_t);
template int launch_special_rows<__nv_bfloat16>(const AttnArgs&, cudaStream_t);

}  // namespace zebra
