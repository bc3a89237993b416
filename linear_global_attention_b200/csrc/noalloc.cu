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

// Device address of the scratch area on the current device, resolved on the
// first call on that device and cached for the life of the process. A
// cudaDeviceReset destroys the module that holds the array, so the cached
// address is not valid after one (the header says so).
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

}  // namespace zebra

using namespace zebra;

extern "C" int zebra_linear_attn_noalloc(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k,
                                         const void* v, const zebra_layout* layout, const float* A, const float* b,
                                         float rope_base, float eps, void* out, void* stream) {
  // the same argument checks as zebra_linear_attn
  if (int rc = check_geom(g)) return rc;
  if (int rc = check_dtype(dt)) return rc;
  long long ts, hs;
  if (int rc = check_layout(g, dt, layout, &ts, &hs)) return rc;
  if (!(rope_base > 0.f) || !(eps >= 0.f)) {
    set_error("rope_base must be > 0 and eps >= 0");
    return ZEBRA_ERR_INVALID_ARG;
  }
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  if (int rc = check_ptr16(q, "q")) return rc;
  if (int rc = check_ptr16(k, "k")) return rc;
  if (int rc = check_ptr16(v, "v")) return rc;
  if (int rc = check_ptr16(out, "out")) return rc;

  // Scratch layout: per-chunk partials, folded state, bf16 state operand,
  // rotation tables. The token chunks are those of zebra_linear_attn (so the two
  // entry points sum in the same order and agree bit for bit) as long as their
  // partials fit; otherwise the chunks grow until they do.
  const int maxpos = G.Hp > G.Wp ? G.Hp : G.Wp;
  const size_t fixed = align256((size_t)G.H * 64 * 65 * 4) + align256((size_t)G.H * 72 * 64 * 2) +
                       align256((size_t)maxpos * 16 * sizeof(float2)) + align256((size_t)maxpos * 8 * sizeof(float4));
  const size_t per_chunk = (size_t)G.H * 64 * 65 * 4;
  if (fixed + align256(per_chunk) > NOALLOC_BYTES) {
    set_error("this geometry needs more scratch than the built-in 16 MiB area; use zebra_linear_attn");
    return ZEBRA_ERR_UNSUPPORTED;
  }
  int ct_i = 0;
  long long chunks = linear_chunks(G, &ct_i);
  long long ct = ct_i;
  const long long fit = (long long)((NOALLOC_BYTES - fixed - 256) / per_chunk);
  if (chunks > fit) {
    chunks = fit;
    ct = ((G.N + chunks - 1) / chunks + 63) / 64 * 64;
    chunks = (G.N + ct - 1) / ct;
  }
  if (ct > 0x7fffffffLL) {
    set_error("token chunk above 2^31 tokens");
    return ZEBRA_ERR_UNSUPPORTED;
  }
  if (int rc = check_device()) return rc;
  void* base = nullptr;
  if (int rc = noalloc_scratch(&base)) return rc;
  Carver c(base);
  LinearArgs a{};
  a.part = c.take<float>((size_t)chunks * G.H * 64 * 65);
  a.state = c.take<float>((size_t)G.H * 64 * 65);
  a.state_b = c.take<__nv_bfloat16>((size_t)G.H * 72 * 64);
  float2* rope = c.take<float2>((size_t)maxpos * 16);
  float4* rope_g = c.take<float4>((size_t)maxpos * 8);
  if (c.used() > NOALLOC_BYTES) {
    set_error("scratch layout exceeds the built-in area");
    return ZEBRA_ERR_UNSUPPORTED;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int rc = launch_rope_table(rope, rope_g, maxpos, (double)rope_base, st)) return rc;
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
  a.rope_g = rope_g;
  a.maxpos = maxpos;
  a.chunks = (int)chunks;
  a.chunk_tokens = (int)ct;
  a.out = out;
  return dt == ZEBRA_BF16 ? launch_linear<__nv_bfloat16>(a, st) : launch_linear<float>(a, st);
}
