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
// bf16 they run on mma.sync m16n8k16 with fp32 accumulation, 4 warps x 16
// query rows, K/V blocks double-buffered in shared memory by cp.async with an
// XOR swizzle on 16-byte chunks so ldmatrix reads are conflict-free.
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
    const TileShape s = tile_shape(g, u);
    return a.ln_tab[s.rows * s.cols] * LOG2E;
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
// bf16 mma.sync path
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
// round a pair to bf16 in place and return it packed: the softmax sum then uses
// exactly the weights that enter the PV product
__device__ __forceinline__ uint32_t pack_round(float& lo, float& hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  const float2 f = __bfloat1622float2(v);
  lo = f.x;
  hi = f.y;
  return *reinterpret_cast<uint32_t*>(&v);
}

// byte offset of (row, 16-byte chunk) in a swizzled 64x64 bf16 tile
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

struct MmaSmem {
  __nv_bfloat16 q[64 * 64];
  __nv_bfloat16 k[2][64 * 64];
  __nv_bfloat16 v[2][64 * 64];
  float bias[2][64];
};

// Dense rows of the special-token queries (mma.sync, bf16): CTA = one block of
// 64 special queries x one head x one key split (blockIdx.z of a.splits); the
// key range is the split's share of the patch tiles, plus every special key in
// split 0. Writes unnormalised partial O, row maximum and row sum for
// special_combine_kernel. (MODE 1 is the only mode: the sparse patch rows run
// on the tcgen05 kernel.)
template <int MODE>
__global__ void __launch_bounds__(128) attn_mma_kernel(const __grid_constant__ AttnArgs a) {
  static_assert(MODE == 1, "dense special-token rows only");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  MmaSmem& sm = *reinterpret_cast<MmaSmem*>(smem_raw);
  const Geo& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int t = blockIdx.x;  // special query block

  // query rows -> shared (swizzled)
  const __nv_bfloat16* qsrc = static_cast<const __nv_bfloat16*>(a.Qs) + ((size_t)h * g.NSp + (size_t)t * 64) * D;
  for (int i = tid; i < 512; i += 128) {
    const int r = i >> 3, c = i & 7;
    cp_async16(smem_u32(sm.q) + swz(r, c), qsrc + r * D + c * 8);
  }
  cp_async_commit();

  BlockIter it{};
  it.phase = 0;
  const int sp = blockIdx.z;
  it.w = (int)((long long)g.T * sp / a.splits);
  it.t_end = (int)((long long)g.T * (sp + 1) / a.splits);
  const bool with_special = sp == 0;

  auto issue = [&](int kind, int id, int buf) {
    const __nv_bfloat16 *ks, *vs;
    block_src<__nv_bfloat16>(a, h, kind, id, ks, vs);
    for (int i = tid; i < 512; i += 128) {
      const int r = i >> 3, c = i & 7;
      cp_async16(smem_u32(sm.k[buf]) + swz(r, c), ks + r * D + c * 8);
      cp_async16(smem_u32(sm.v[buf]) + swz(r, c), vs + r * D + c * 8);
    }
    if (tid < 64) sm.bias[buf][tid] = block_bias(a, nullptr, t, kind, id, tid);   // kinds 0 and 2 only
  };

  int kind = 0, id = 0, nv = 0;
  long long keys = 0;  // visible keys per query row, summed over blocks
  bool have = next_block_dense(it, g, with_special, kind, id, nv);
  if (have) {
    issue(kind, id, 0);
    keys += nv;
  }
  cp_async_commit();

  const float sc = LOG2E * 0.125f;  // log2(e) / sqrt(64)
  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  uint32_t qf[4][4];
  bool qloaded = false;
  const int g4 = lane >> 2, q4 = lane & 3;

  int buf = 0;
  while (have) {
    int nkind = 0, nid = 0, nnv = 0;
    const bool nhave = next_block_dense(it, g, with_special, nkind, nid, nnv);
    if (nhave) {
      issue(nkind, nid, buf ^ 1);
      keys += nnv;
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (!qloaded) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int mi = lane >> 3, ri = lane & 7;
        const int row = warp * 16 + (mi & 1) * 8 + ri;
        ldsm_x4(smem_u32(sm.q) + swz(row, 2 * ks + (mi >> 1)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
      qloaded = true;
    }
    // S = Q K^T
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t kb = smem_u32(sm.k[buf]);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int mi = lane >> 3, ri = lane & 7;
        const int row = np * 16 + (mi >> 1) * 8 + ri;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz(row, 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
    }
    // online softmax (rows g4 and g4 + 8 of this warp)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float b0v = sm.bias[buf][8 * j + 2 * q4], b1v = sm.bias[buf][8 * j + 2 * q4 + 1];
      s[j][0] = fmaf(s[j][0], sc, b0v);
      s[j][1] = fmaf(s[j][1], sc, b1v);
      s[j][2] = fmaf(s[j][2], sc, b0v);
      s[j][3] = fmaf(s[j][3], sc, b1v);
      mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
      mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = fast_exp2(m0 - base0), al1 = fast_exp2(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pk[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      s[j][0] = fast_exp2(s[j][0] - base0);
      s[j][1] = fast_exp2(s[j][1] - base0);
      s[j][2] = fast_exp2(s[j][2] - base1);
      s[j][3] = fast_exp2(s[j][3] - base1);
      pk[j][0] = pack_round(s[j][0], s[j][1]);
      pk[j][1] = pack_round(s[j][2], s[j][3]);
      rs0 += s[j][0] + s[j][1];
      rs1 += s[j][2] + s[j][3];
    }
    l0 = l0 * al0 + rs0;
    l1 = l1 * al1 + rs1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      o[j][0] *= al0; o[j][1] *= al0;
      o[j][2] *= al1; o[j][3] *= al1;
    }
    // O += P V
    const uint32_t vb = smem_u32(sm.v[buf]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pk[2 * kk][0];
      pa[1] = pk[2 * kk][1];
      pa[2] = pk[2 * kk + 1][0];
      pa[3] = pk[2 * kk + 1][1];
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        const int mi = lane >> 3, ri = lane & 7;
        const int row = kk * 16 + (mi & 1) * 8 + ri;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz(row, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa, b0, b1);
        mma_bf16(o[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncthreads();
    buf ^= 1;
    have = nhave;
    kind = nkind;
    id = nid;
  }
  cp_async_wait<0>();
  if (!qloaded) __syncthreads();
  if (tid == 0) {
    const long long rows = min(64, g.NS - t * 64);
    atomicAdd(&g_logits[1], (unsigned long long)(rows * keys));
  }

  const int r0 = warp * 16 + g4, r1 = r0 + 8;
  {
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = half ? r1 : r0;
      const int qi = t * 64 + r;  // special query index
      const size_t row = ((size_t)sp * g.H + h) * g.NSp + qi;
      float* po = a.part_o + row * D;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = 8 * j + 2 * q4;
        *reinterpret_cast<float2*>(po + c) = make_float2(o[j][half * 2], o[j][half * 2 + 1]);
      }
      if (q4 == 0) *reinterpret_cast<float2*>(a.part_ml + row * 2) = make_float2(half ? m1 : m0, half ? l1 : l0);
    }
  }
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
  dim3 grid(a.g.NSp / 64, a.g.H, a.splits);
  {
  ProfScope prof("attn_special_rows", st);
  if (sizeof(T) == 2) {
    const size_t smem = sizeof(MmaSmem);
    cudaFuncSetAttribute(attn_mma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_mma_kernel<1><<<grid, 128, smem, st>>>(a);
  } else {
    attn_simt_kernel<1><<<grid, 64, 0, st>>>(a);
  }
  }
  count_launch();
  int rc = check_launch("attn_kernel<special rows>");
  if (rc) return rc;
  const long long threads = (long long)a.g.NS * a.g.H * 32;
  ProfScope prof("special_combine", st);
  special_combine_kernel<T><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(a);
  count_launch();
  return check_launch("special_combine_kernel");
}

template int launch_special_rows<float>(const AttnArgs&, cudaStream_t);
template int launch_special_rows<__nv_bfloat16>(const AttnArgs&, cudaStream_t);

}  // namespace zebra
