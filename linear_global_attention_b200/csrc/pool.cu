// Tile mean-pooling and tile-major packing.
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views":
//  - section "Linear-centered stages plus tile-sparse stages": omitted tiles are
//    summarised by mean key/value landmarks; the mean-pooled query and key of a
//    tile also feed the selector;
//  - section "Speedup scales with the number of input views": keys and values
//    are packed into tile-major order for the sparse stage.
//
// One CTA pools one tile for a group of heads of up to three tensors (Q, K, V:
// blockIdx.z). Each thread owns 16 bytes (8 bf16 / 4 fp32 channels) of one
// head and walks the tile's tokens, so a warp reads whole 128-byte head rows
// and consecutive heads of a token are contiguous: every load is a coalesced
// 16-byte vector load. The same pass writes the packed tile rows (zero-padded
// to 64, or for K and V of the tcgen05 kernel to a multiple of 8 in the dense
// layout) and, at the end, the fp32 mean and its landmark copy.
//
// Optional prologue (stacked sparse/dense layers): RMS-normalise each head row
// (x / sqrt(mean(x^2) + eps)) and turn channel pairs (j, j+16) of channels 0-31
// by patch row and of channels 32-63 by patch column (2D rotary positions,
// angle pos * base^(-j/16), cos/sin from a table). The 8 (or 16) threads of a
// head exchange partial sums and rotation partners with warp shuffles.
#include "common.cuh"
#include "kernels.cuh"

namespace zebra {

template <typename T>
__device__ __forceinline__ void norm_rope_chunk(float* x, int chunk, bool rope, int row, int col,
                                                const float2* __restrict__ tab, float eps) {
  constexpr int P = Elem<T>::PER16;
  constexpr int CPT = D / P;
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < P; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int o = 1; o < CPT; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float sc = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
  for (int e = 0; e < P; ++e) x[e] *= sc;
  float part[P];
#pragma unroll
  for (int e = 0; e < P; ++e) part[e] = __shfl_xor_sync(0xffffffffu, x[e], 16 / P);
  if (rope) {
    const int c0 = chunk * P;
    const int pos = c0 < 32 ? row : col;
    const bool first = (c0 & 16) == 0;
#pragma unroll
    for (int e = 0; e < P; ++e) {
      const float2 cs = tab[pos * 16 + ((c0 + e) & 15)];
      x[e] = first ? fmaf(x[e], cs.x, -part[e] * cs.y) : fmaf(x[e], cs.x, part[e] * cs.y);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) pool_pack_kernel(PoolArgs<T> a) {
  constexpr int P = Elem<T>::PER16;
  constexpr int CPT = D / P;
  constexpr int HPC = 128 / CPT;
  const Geo& g = a.g;
  const int u = blockIdx.x;
  const int z = blockIdx.z;
  const T* __restrict__ x = a.x[z];
  if (x == nullptr) return;
  const int chunk = threadIdx.x % CPT;
  const int h = blockIdx.y * HPC + threadIdx.x / CPT;
  const bool hv = h < g.H;
  const int hh = hv ? h : 0;
  if (u >= g.T) {  // padding landmark rows T..Tpad-1 are zero
    if (hv && a.lmk[z]) store16_zero(a.lmk[z] + ((size_t)hh * g.Tpad + u) * D + chunk * P);
    return;
  }
  const TileShape s = tile_shape(g, u);
  const int n = s.rows * s.cols;
  const bool nr = a.norm_rope[z] != 0;
  const bool dense = a.dense_kv && z > 0;
  const size_t prow = dense ? (size_t)hh * g.V * g.RPV + dense_tile_row(g, u) : ((size_t)hh * g.T + u) * TOK;
  T* packed = a.packed[z] ? a.packed[z] + prow * D + chunk * P : nullptr;
  const int pad_to = dense ? (n + 7) & ~7 : TOK;   // zero rows after the tile's n rows

  float sum[P];
#pragma unroll
  for (int e = 0; e < P; ++e) sum[e] = 0.f;

  for (int a0 = 0; a0 < n; a0 += 4) {
    float v[4][P];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = a0 + i;
      if (r < n) {
        const long long tok = tile_token(g, s, r);
        load16(x + tok * a.ts + (long long)hh * a.hs + chunk * P, v[i]);
      } else {
#pragma unroll
        for (int e = 0; e < P; ++e) v[i][e] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = a0 + i;
      if (nr && r < n) {   // uniform across the warp: r < n is the same for all lanes
        const int rr = r / s.cols;
        norm_rope_chunk<T>(v[i], chunk, a.rope != nullptr, s.r0 + rr, s.c0 + (r - rr * s.cols), a.rope, a.eps);
      }
      if (r < n) {
#pragma unroll
        for (int e = 0; e < P; ++e) sum[e] += v[i][e];
        if (packed && hv) store16(packed + (size_t)r * D, v[i]);
      }
    }
  }
  if (packed && hv)
    for (int r = n; r < pad_to; ++r) store16_zero(packed + (size_t)r * D);
  if (!hv) return;
  const float inv = 1.0f / (float)n;
#pragma unroll
  for (int e = 0; e < P; ++e) sum[e] *= inv;
  if (a.mean[z]) {
    float* m = a.mean[z] + ((size_t)hh * g.T + u) * D + chunk * P;
#pragma unroll
    for (int e = 0; e < P; e += 4) *reinterpret_cast<float4*>(m + e) = make_float4(sum[e], sum[e + 1], sum[e + 2], sum[e + 3]);
  }
  if (a.lmk[z]) store16(a.lmk[z] + ((size_t)hh * g.Tpad + u) * D + chunk * P, sum);
  if (a.counts && z == 0 && h == 0 && chunk == 0) a.counts[u] = n;
  if (a.lmk_bias && z == 0 && h == 0 && chunk == 0) a.lmk_bias[u] = a.ln_tab[n] * LOG2E;
}

// Special tokens of all views, packed per head: out[h][i][:] for i < NSp
// (zero rows for i >= NS). Optional RMS norm (no rotation: special tokens carry
// no patch position).
template <typename T>
__global__ void __launch_bounds__(128) pack_special_kernel(SpecialArgs<T> a) {
  constexpr int P = Elem<T>::PER16;
  constexpr int CPT = D / P;
  const Geo& g = a.g;
  const int z = blockIdx.z;
  if (a.x[z] == nullptr) return;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int chunk = (int)(gid % CPT);
  const long long ih = gid / CPT;               // (i, h) flattened, h fastest
  const long long total = (long long)g.NSp * g.H;
  const bool valid = ih < total;
  const int h = valid ? (int)(ih % g.H) : 0;
  const int i = valid ? (int)(ih / g.H) : 0;
  float v[P];
  const bool real = valid && i < g.NS;
  if (real) {
    load16(a.x[z] + special_token(g, i) * a.ts + (long long)h * a.hs + chunk * P, v);
  } else {
#pragma unroll
    for (int e = 0; e < P; ++e) v[e] = 0.f;
  }
  if (a.norm[z]) {
    // all CPT lanes of an (i, h) group are valid or invalid together
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < P; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
    for (int o = 1; o < CPT; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float sc = real ? rsqrtf(ss * (1.0f / D) + a.eps) : 0.f;
#pragma unroll
    for (int e = 0; e < P; ++e) v[e] *= sc;
  }
  if (valid) store16(a.out[z] + ((size_t)h * g.NSp + i) * D + chunk * P, v);
}

// cos/sin table of the 2D rotation: tab[pos*16 + j] = (cos, sin)(pos * base^(-j/16)),
// evaluated in double precision. tab_g (optional) holds the same values as the
// packed-pair operands of the linear kernels, group i of the pairs j = 2i,
// 2i + 1 before position: tab_g[i*maxpos + pos] = (cos_j, cos_j+1, sin_j, sin_j+1).
__global__ void rope_table_kernel(float2* tab, float4* tab_g, int maxpos, double base) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= maxpos * 16) return;
  const int pos = i / 16, j = i % 16;
  const double ang = (double)pos * pow(base, -(double)j / 16.0);
  const float c = (float)cos(ang), s = (float)sin(ang);
  tab[i] = make_float2(c, s);
  if (tab_g) {
    float* g = reinterpret_cast<float*>(tab_g + (size_t)(j / 2) * maxpos + pos);
    g[j & 1] = c;
    g[2 + (j & 1)] = s;
  }
}

template <typename T>
int launch_pool_pack(const PoolArgs<T>& a, int ntensors, cudaStream_t st) {
  if (a.g.T == 0) return ZEBRA_OK;
  constexpr int HPC = 128 / (D / Elem<T>::PER16);
  dim3 grid(a.g.Tpad, (a.g.H + HPC - 1) / HPC, ntensors);
  ProfScope prof("pool_pack", st);
  pool_pack_kernel<T><<<grid, 128, 0, st>>>(a);
  count_launch();
  return check_launch("pool_pack_kernel");
}

template <typename T>
int launch_pack_special(const SpecialArgs<T>& a, int ntensors, cudaStream_t st) {
  const long long threads = (long long)a.g.NSp * a.g.H * (D / Elem<T>::PER16);
  if (threads == 0) return ZEBRA_OK;
  dim3 grid((unsigned)((threads + 127) / 128), 1, ntensors);
  ProfScope prof("pack_special", st);
  pack_special_kernel<T><<<grid, 128, 0, st>>>(a);
  count_launch();
  return check_launch("pack_special_kernel");
}

int launch_rope_table(float2* tab, float4* tab_g, int maxpos, double base, cudaStream_t st) {
  const int n = maxpos * 16;
  ProfScope prof("rope_table", st);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(tab, tab_g, maxpos, base);
  count_launch();
  return check_launch("rope_table_kernel");
}

template int launch_pool_pack<float>(const PoolArgs<float>&, int, cudaStream_t);
template int launch_pool_pack<__nv_bfloat16>(const PoolArgs<__nv_bfloat16>&, int, cudaStream_t);
template int launch_pack_special<float>(const SpecialArgs<float>&, int, cudaStream_t);
template int launch_pack_special<__nv_bfloat16>(const SpecialArgs<__nv_bfloat16>&, int, cudaStream_t);

}  // namespace zebra
