// Linear stage without a caller workspace: the scratch lives in a fixed
// device array built into the library (see zebra_linear_attn_noalloc in
// include/zebra.h). The computation is the same as zebra_linear_attn; only the
// origin of the scratch memory differs.
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.cuh"

namespace zebra {

// Built-in scratch area. Every device that loads the library holds one copy
// until the process exits. Host code must not use the symbol as an address: it
// resolves the device address with cudaGetSymbolAddress, once per device.
constexpr size_t NOALLOC_BYTES = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_BYTES];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch area on the current device (resolved on first use).
static int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    set_error(std::string("no CUDA device: ") + cudaGetErrorString(e));
    return ZEBRA_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    set_error("device ordinal above 63");
    return ZEBRA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      set_error(std::string("cudaGetSymbolAddress of the built-in scratch failed: ") + cudaGetErrorString(e));
      return ZEBRA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ZEBRA_OK;
}

static int na_fail(int code, const std::string& msg) {
  set_error(msg);
  return code;
}

}  // namespace zebra

using namespace zebra;

extern "C" int zebra_linear_attn_noalloc(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k,
                                         const void* v, const zebra_layout* layout, const float* A, const float* b,
                                         float rope_base, float eps, void* out, void* stream) {
  if (!g) return na_fail(ZEBRA_ERR_INVALID_ARG, "geometry pointer is null");
  if (g->head_dim != 64) return na_fail(ZEBRA_ERR_UNSUPPORTED, "head_dim must be 64");
  if (g->tile != 8) return na_fail(ZEBRA_ERR_UNSUPPORTED, "tile must be 8");
  if (g->views < 0 || g->grid_h < 1 || g->grid_w < 1 || g->heads < 1 || g->n_special < 0 || g->n_special > 64 ||
      g->grid_h > 4096 || g->grid_w > 4096)
    return na_fail(ZEBRA_ERR_INVALID_ARG, "invalid geometry");
  if (dt != ZEBRA_F32 && dt != ZEBRA_BF16) return na_fail(ZEBRA_ERR_INVALID_ARG, "unknown dtype");
  if (!(rope_base > 0.f) || !(eps >= 0.f)) return na_fail(ZEBRA_ERR_INVALID_ARG, "rope_base must be > 0 and eps >= 0");
  const long long ts = layout ? layout->tok_stride : (long long)g->heads * 64;
  const long long hs = layout ? layout->head_stride : 64;
  const long long vec = dt == ZEBRA_BF16 ? 8 : 4;
  if (ts < 0 || hs < 0 || ts % vec || hs % vec)
    return na_fail(ZEBRA_ERR_INVALID_ARG, "strides must be non-negative multiples of 16 bytes");
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  for (const void* p : {q, k, v, static_cast<const void*>(out)})
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15))
      return na_fail(ZEBRA_ERR_INVALID_ARG, "q, k, v and out must be non-null and 16-byte aligned");

  // carve: per-chunk partials, folded state, bf16 state operand, rotation table
  const int maxpos = G.Hp > G.Wp ? G.Hp : G.Wp;
  const size_t fixed = align256((size_t)G.H * 64 * 65 * 4) + align256((size_t)G.H * 72 * 64 * 2) +
                       align256((size_t)maxpos * 16 * sizeof(float2));
  const size_t per_chunk = (size_t)G.H * 64 * 65 * 4;
  if (fixed + align256(per_chunk) > NOALLOC_BYTES)
    return na_fail(ZEBRA_ERR_UNSUPPORTED,
                   "this geometry needs more scratch than the built-in 16 MiB area; use zebra_linear_attn");
  long long chunks = (G.N + 2047) / 2048;
  const long long fit = (long long)((NOALLOC_BYTES - fixed - 256) / per_chunk);
  if (chunks > 32) chunks = 32;
  if (chunks > fit) chunks = fit;
  if (chunks < 1) chunks = 1;
  long long ct = ((G.N + chunks - 1) / chunks + 63) / 64 * 64;
  chunks = (G.N + ct - 1) / ct;

  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return na_fail(ZEBRA_ERR_CUDA, "no CUDA device");
  }
  if (major != 10) return na_fail(ZEBRA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200)");
  void* base = nullptr;
  if (int rc = noalloc_scratch(&base)) return rc;
  Carver c(base);
  LinearArgs a{};
  a.part = c.take<float>((size_t)chunks * G.H * 64 * 65);
  a.state = c.take<float>((size_t)G.H * 64 * 65);
  a.state_b = c.take<__nv_bfloat16>((size_t)G.H * 72 * 64);
  float2* rope = c.take<float2>((size_t)maxpos * 16);
  if (c.used() > NOALLOC_BYTES) return na_fail(ZEBRA_ERR_UNSUPPORTED, "scratch layout exceeds the built-in area");

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int rc = launch_rope_table(rope, maxpos, (double)rope_base, st)) return rc;
  a.g = G;
  a.q = q;
  a.k = k;
  a.v = v;
  a.ts = ts;
  a.hs = hs;
  a.A = A;
  a.b = b;
  a.eps = eps;
  a.rope = rope;
  a.chunks = (int)chunks;
  a.chunk_tokens = (int)ct;
  a.out = out;
  return dt == ZEBRA_BF16 ? launch_linear<__nv_bfloat16>(a, st) : launch_linear<float>(a, st);
}
