// Shared device/host helpers of the Zebra3D global-attention library.
//
// Token layout and tile partition follow the page "How Hybrid Attention Lets
// Feed-Forward 3D Models Scale to Many Views", section "Linear-centered stages
// plus tile-sparse stages" (8x8-patch tiles of 64 tokens per image; special
// tokens per view), with partial bottom/right edge tiles.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "zebra.h"

namespace zebra {

constexpr int D = 64;      // head dimension (the only one supported)
constexpr int TILE = 8;    // tile side in patches
constexpr int TOK = 64;    // tokens in a complete tile / rows of a packed block

// ---------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------
// Division by a fixed divisor d >= 1 as a multiply and a shift, exact for
// dividends in [0, 2^31): with s = ceil(log2 d) and m = ceil(2^(31+s) / d),
// m < 2^32 and m d - 2^(31+s) < d <= 2^s, so n m / 2^(31+s) exceeds n / d by
// less than 1/d and its floor is floor(n / d).
struct FastDiv {
  uint32_t m;
  int s;   // 0 for d = 1
};
inline FastDiv make_fastdiv(uint32_t d) {
  int s = 0;
  while ((1ull << s) < d) ++s;
  if (s == 0) return FastDiv{0u, 0};
  const unsigned long long m = ((1ull << (31 + s)) + d - 1) / d;
  return FastDiv{(uint32_t)m, s};
}
__host__ __device__ __forceinline__ int fdiv(int n, FastDiv f) {
  if (f.s == 0) return n;
#ifdef __CUDA_ARCH__
  return (int)(__umulhi((uint32_t)n, f.m) >> (f.s - 1));
#else
  return (int)((((unsigned long long)(uint32_t)n * f.m) >> 32) >> (f.s - 1));
#endif
}

struct Geo {
  int V, Hp, Wp, S, H;   // views, grid rows, grid cols, special tokens/view, heads
  int L;                 // tokens per view
  int Tr, Tc, Tv, T;     // tile rows/cols per view, tiles per view, tiles
  int W;                 // 32-bit mask words per selection row
  int NS, NSp;           // special tokens (all views), padded to a multiple of 64
  int Tpad;              // T padded to a multiple of 64
  long long N;           // tokens
  FastDiv fTv, fTc;      // division by Tv and Tc
  FastDiv fL, fWp;       // division by L and Wp
  int RPV;               // rows per view of the 8-row-granular dense K/V layout (dense_tile_row)
};

inline Geo make_geo(const zebra_geom& g) {
  Geo o;
  o.V = g.views; o.Hp = g.grid_h; o.Wp = g.grid_w; o.S = g.n_special; o.H = g.heads;
  o.L = o.S + o.Hp * o.Wp;
  o.Tr = (o.Hp + TILE - 1) / TILE;
  o.Tc = (o.Wp + TILE - 1) / TILE;
  o.Tv = o.Tr * o.Tc;
  o.T = o.V * o.Tv;
  o.W = (o.T + 31) / 32;
  o.NS = o.S * o.V;
  o.NSp = (o.NS + 63) / 64 * 64;
  o.Tpad = (o.T + 63) / 64 * 64;
  o.N = (long long)o.V * o.L;
  o.fTv = make_fastdiv((uint32_t)(o.Tv > 0 ? o.Tv : 1));
  o.fTc = make_fastdiv((uint32_t)(o.Tc > 0 ? o.Tc : 1));
  o.fL = make_fastdiv((uint32_t)(o.L > 0 ? o.L : 1));
  o.fWp = make_fastdiv((uint32_t)(o.Wp > 0 ? o.Wp : 1));
  {
    // every tile but the corner one holds a multiple of 8 tokens (8 x cols or rows x 8)
    const int rl = o.Hp - TILE * (o.Tr - 1), cl = o.Wp - TILE * (o.Tc - 1);
    o.RPV = TILE * o.Wp * (o.Tr - 1) + rl * TILE * (o.Tc - 1) + ((rl * cl + 7) & ~7);
  }
  return o;
}

struct TileShape {
  int view, r0, c0, rows, cols;
};

__host__ __device__ __forceinline__ TileShape tile_shape(const Geo& g, int u) {
  TileShape s;
  s.view = fdiv(u, g.fTv);
  int p = u - s.view * g.Tv;
  int br = fdiv(p, g.fTc), bc = p - br * g.Tc;
  s.r0 = br * TILE;
  s.c0 = bc * TILE;
  s.rows = min(TILE, g.Hp - s.r0);
  s.cols = min(TILE, g.Wp - s.c0);
  return s;
}

// Dense K/V layout of the tcgen05 sparse kernel: per head, the tiles of each
// view in order, each tile's rows (row-major inside the tile) followed by zero
// rows up to a multiple of 8 (only the corner tile of a view needs them). Tile
// u starts at row dense_tile_row(g, u) of its head; a head holds V * RPV rows.
// All tiles before row band br of a view are full 8-row bands (8 * Wp tokens
// each), and the tiles before column bc in band br have 8 columns each.
__host__ __device__ __forceinline__ int dense_tile_row(const Geo& g, int u) {
  const int view = fdiv(u, g.fTv);
  const int p = u - view * g.Tv;
  const int br = fdiv(p, g.fTc), bc = p - br * g.Tc;
  const int rows = min(TILE, g.Hp - br * TILE);
  return view * g.RPV + TILE * g.Wp * br + rows * TILE * bc;
}

// token index of row a (row-major inside the tile) of tile shape s
__host__ __device__ __forceinline__ long long tile_token(const Geo& g, const TileShape& s, int a) {
  int rr = a / s.cols, cc = a - rr * s.cols;
  return (long long)s.view * g.L + g.S + (long long)(s.r0 + rr) * g.Wp + (s.c0 + cc);
}

// token index of special token number i (0 <= i < NS): view i / S, slot i % S
__host__ __device__ __forceinline__ long long special_token(const Geo& g, int i) {
  int v = i / g.S;
  return (long long)v * g.L + (i - v * g.S);
}

// ---------------------------------------------------------------------------
// element helpers
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int PER16 = 4;  // elements per 16 bytes
  __device__ static float to_f(float x) { return x; }
  __device__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int PER16 = 8;
  __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// load 16 bytes as PER16 floats
__device__ __forceinline__ void load16(const float* p, float* o) {
  float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* o) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x; o[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store16(float* p, const float* o) {
  *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* o) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = v;
}
__device__ __forceinline__ void store16_zero(void* p) { *reinterpret_cast<uint4*>(p) = make_uint4(0, 0, 0, 0); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float LOG2E = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// host-side plumbing shared by the translation units
// ---------------------------------------------------------------------------
void set_error(const std::string& msg);
void count_launch(int n = 1);
int check_launch(const char* what);   // ZEBRA_OK or ZEBRA_ERR_CUDA (sets the message)

// Argument checks shared by the entry points (each returns a ZEBRA_* status and
// sets the message): geometry limits, element type, strides of a [N, H, d]
// input (NULL layout = contiguous; fills *ts, *hs), a non-null 16-byte aligned
// device pointer, and an sm_100 current device.
int check_geom(const zebra_geom* g);
int check_dtype(zebra_dtype dt);
int check_layout(const zebra_geom* g, zebra_dtype dt, const zebra_layout* lay, long long* ts, long long* hs);
int check_ptr16(const void* p, const char* name);
int check_device();

// Optional per-kernel timing: while profiling is on (zebra_profile_enable), a
// ProfScope records a CUDA event on `st` when it is made and another when it
// goes out of scope, around one kernel launch (or set_launches(n) launches).
struct ProfScope {
  int slot = -1;
  cudaStream_t st;
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  void set_launches(int n);
};

// visible-logit counters of the attention kernels (per device): [0] patch rows
// of the sparse kernel, [1] special-token rows
void reset_logit_counters();
void read_logit_counters(unsigned long long* out2);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Bump allocator over the caller's workspace.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T> T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align256(count * sizeof(T));
    return p;
  }
  size_t used() const { return off; }
};

}  // namespace zebra
