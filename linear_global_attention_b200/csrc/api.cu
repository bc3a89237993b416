// C ABI of the Zebra3D global-attention library: argument validation,
// workspace carving and kernel orchestration. See include/zebra.h for the
// contract of every entry point.
#include <type_traits>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"

namespace zebra {

static thread_local std::string g_err;
static std::atomic<unsigned long long> g_launches{0};

void set_error(const std::string& msg) { g_err = msg; }
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// ---- profiling records ----
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
  int launches;
};
static std::mutex g_prof_mu;
static std::atomic<bool> g_prof_on{false};
static std::vector<ProfRec> g_recs;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

ProfScope::ProfScope(const char* name, cudaStream_t s) : st(s) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRec r{name, take_event(), take_event(), 1};
  cudaEventRecord(r.a, st);
  slot = (int)g_recs.size();
  g_recs.push_back(r);
}

ProfScope::~ProfScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEventRecord(g_recs[slot].b, st);
}

void ProfScope::set_launches(int n) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_recs[slot].launches = n;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(std::string(what) + ": " + cudaGetErrorString(e));
    return ZEBRA_ERR_CUDA;
  }
  return ZEBRA_OK;
}

static int fail(int code, const std::string& msg) {
  set_error(msg);
  return code;
}

int check_geom(const zebra_geom* g) {
  if (!g) return fail(ZEBRA_ERR_INVALID_ARG, "geometry pointer is null");
  if (g->head_dim != 64) return fail(ZEBRA_ERR_UNSUPPORTED, "head_dim must be 64");
  if (g->tile != 8) return fail(ZEBRA_ERR_UNSUPPORTED, "tile must be 8");
  if (g->views < 0) return fail(ZEBRA_ERR_INVALID_ARG, "views must be >= 0");
  if (g->grid_h < 1 || g->grid_w < 1) return fail(ZEBRA_ERR_INVALID_ARG, "grid_h and grid_w must be >= 1");
  if (g->heads < 1) return fail(ZEBRA_ERR_INVALID_ARG, "heads must be >= 1");
  if (g->n_special < 0 || g->n_special > 64) return fail(ZEBRA_ERR_INVALID_ARG, "n_special must lie in [0, 64]");
  if (g->grid_h > 4096 || g->grid_w > 4096) return fail(ZEBRA_ERR_UNSUPPORTED, "grid sides above 4096");
  const long long tv = (long long)((g->grid_h + 7) / 8) * ((g->grid_w + 7) / 8);
  const long long L = (long long)g->n_special + (long long)g->grid_h * g->grid_w;
  if ((long long)g->views * tv > (1LL << 30)) return fail(ZEBRA_ERR_UNSUPPORTED, "too many tiles");
  if ((long long)g->views * L * g->heads > (1LL << 40)) return fail(ZEBRA_ERR_UNSUPPORTED, "too many tokens");
  return ZEBRA_OK;
}

static int check_y(double y) {
  if (!(y >= 0.0 && y < 1.0)) return fail(ZEBRA_ERR_INVALID_ARG, "y must lie in [0, 1)");
  return ZEBRA_OK;
}

int check_dtype(zebra_dtype dt) {
  if (dt != ZEBRA_F32 && dt != ZEBRA_BF16) return fail(ZEBRA_ERR_INVALID_ARG, "unknown dtype");
  return ZEBRA_OK;
}

static size_t esize(zebra_dtype dt) { return dt == ZEBRA_BF16 ? 2 : 4; }

int check_layout(const zebra_geom* g, zebra_dtype dt, const zebra_layout* lay, long long* ts, long long* hs) {
  const long long H = g->heads;
  *ts = lay ? lay->tok_stride : H * 64;
  *hs = lay ? lay->head_stride : 64;
  const long long vec = 16 / (long long)esize(dt);
  if (*ts < 0 || *hs < 0) return fail(ZEBRA_ERR_INVALID_ARG, "strides must be non-negative");
  if (*ts % vec || *hs % vec) return fail(ZEBRA_ERR_INVALID_ARG, "strides must be multiples of 16 bytes");
  return ZEBRA_OK;
}

// Workspaces are carved into 256-byte-aligned pieces that TMA and 16-byte
// asynchronous copies read, so the base must be 256-byte aligned (cudaMalloc's are).
static int check_workspace(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return fail(ZEBRA_ERR_WORKSPACE, "workspace too small");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(ZEBRA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  return ZEBRA_OK;
}

int check_ptr16(const void* p, const char* name) {
  if (!p) return fail(ZEBRA_ERR_INVALID_ARG, std::string(name) + " is null");
  if (reinterpret_cast<uintptr_t>(p) & 15) return fail(ZEBRA_ERR_INVALID_ARG, std::string(name) + " must be 16-byte aligned");
  return ZEBRA_OK;
}

// current device must be an sm_100 part
int check_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ZEBRA_ERR_CUDA, std::string("no CUDA device: ") + cudaGetErrorString(e));
  }
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return fail(ZEBRA_ERR_CUDA, cudaGetErrorString(e));
  if (major != 10) return fail(ZEBRA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200)");
  return ZEBRA_OK;
}

#define ZTRY(expr)          \
  do {                      \
    int _rc = (expr);       \
    if (_rc) return _rc;    \
  } while (0)

// ---------------------------------------------------------------------------
// workspace layouts
// ---------------------------------------------------------------------------
static int max_pos(const Geo& G) { return G.Hp > G.Wp ? G.Hp : G.Wp; }

struct SelectWs {
  float* scores;
  int hc, Tld;
  void *qsplit, *ksplit, *gemm_ws;
};
static void carve_select(const Geo& G, Carver& c, SelectWs& w) {
  w.Tld = (G.T + 3) / 4 * 4;
  const size_t per_head = (size_t)G.T * w.Tld * 4;
  const size_t budget = size_t(4) << 30;
  long long hc = per_head ? (long long)(budget / per_head) : G.H;
  if (hc < 1) hc = 1;
  if (hc > G.H) hc = G.H;
  w.hc = (int)hc;
  w.scores = c.take<float>((size_t)w.hc * G.T * w.Tld);
  w.qsplit = c.take<__nv_bfloat16>((size_t)w.hc * G.T * SPLIT_K);
  w.ksplit = c.take<__nv_bfloat16>((size_t)w.hc * G.T * SPLIT_K);
  w.gemm_ws = c.take<char>(GEMM_WS_BYTES);
}

struct SparseWs {
  void *Qp, *Kp, *Vp, *Qs, *Ks, *Vs, *Kl, *Vl;
  float *qm, *km, *vm;
  uint32_t* mask;
  SelectWs sel;
  float *part_o, *part_ml;
  int splits;
  float2* rope;
  float* lmk_bias;
};
static void carve_sparse(const Geo& G, zebra_dtype dt, Carver& c, SparseWs& w) {
  const size_t es = esize(dt);
  const size_t packed = (size_t)G.H * G.T * TOK * D * es;
  const size_t spec = (size_t)G.H * G.NSp * D * es;
  const size_t lmk = (size_t)G.H * G.Tpad * D * es;
  const size_t means = (size_t)G.H * G.T * D;
  w.Qp = c.take<char>(packed);
  w.Kp = c.take<char>(packed);
  w.Vp = c.take<char>(packed);
  w.Qs = c.take<char>(spec);
  w.Ks = c.take<char>(spec);
  w.Vs = c.take<char>(spec);
  w.Kl = c.take<char>(lmk);
  w.Vl = c.take<char>(lmk);
  w.qm = c.take<float>(means);
  w.km = c.take<float>(means);
  w.vm = c.take<float>(means);
  w.mask = c.take<uint32_t>((size_t)G.H * G.T * G.W);
  w.lmk_bias = c.take<float>((size_t)G.T);
  carve_select(G, c, w.sel);
  // key splits of the special-token rows: about 8 resident waves of work
  // items (148 SMs x 4 CTAs each) over all query blocks and heads
  const int nqb = G.NSp / 64;
  long long splits = 1;
  if (nqb > 0) {
    splits = (4736 + (long long)nqb * G.H - 1) / ((long long)nqb * G.H);
    if (splits > 64) splits = 64;
    if (splits > G.T) splits = G.T > 0 ? G.T : 1;
    if (splits < 1) splits = 1;
  }
  w.splits = (int)splits;
  w.part_o = c.take<float>((size_t)w.splits * G.H * G.NSp * D);
  w.part_ml = c.take<float>((size_t)w.splits * G.H * G.NSp * 2);
  w.rope = c.take<float2>((size_t)max_pos(G) * 16);
}

struct LinearWs {
  float* part;
  float* state;
  void* state_b;
  float2* rope;
  float4* rope_g;
  int chunks, chunk_tokens;
};
static void carve_linear(const Geo& G, Carver& c, LinearWs& w) {
  w.chunks = linear_chunks(G, &w.chunk_tokens);
  w.part = c.take<float>((size_t)w.chunks * G.H * 64 * 65);
  w.state = c.take<float>((size_t)G.H * 64 * 65);
  w.state_b = c.take<__nv_bfloat16>((size_t)G.H * 72 * 64);
  w.rope = c.take<float2>((size_t)max_pos(G) * 16);
  w.rope_g = c.take<float4>((size_t)max_pos(G) * 8);
}

struct HybridWs {
  void* qkv;
  void* o;
  void* gemm_ws;
  SparseWs sp;
  LinearWs li;
};
static void carve_hybrid(const Geo& G, int kind, Carver& c, HybridWs& w) {
  const size_t Dm = (size_t)G.H * D;
  w.qkv = c.take<__nv_bfloat16>((size_t)G.N * 3 * Dm);
  w.o = c.take<__nv_bfloat16>((size_t)G.N * Dm);
  w.gemm_ws = c.take<char>(GEMM_WS_BYTES);
  if (kind == ZEBRA_LAYER_LINEAR)
    carve_linear(G, c, w.li);
  else
    carve_sparse(G, ZEBRA_BF16, c, w.sp);
}

static void fill_ln_tab(float* tab) {
  tab[0] = 0.f;
  for (int m = 1; m <= TOK; ++m) tab[m] = (float)std::log((double)m);
}

static int keep_of(double y, int T) {
  double k = ceil((1.0 - (double)y) * (double)T - 1e-6);
  if (k < 1) k = 1;
  if (k > T) k = T;
  return (int)k;
}

// ---------------------------------------------------------------------------
// internal stage runners (arguments already validated)
// ---------------------------------------------------------------------------
static int run_select(const Geo& G, const float* qm, const float* km, int keep, uint32_t* mask, uint8_t* near_tie,
                      const SelectWs& w, cudaStream_t st) {
  if (G.T > SELECT_MAX_T) return fail(ZEBRA_ERR_UNSUPPORTED, "selection supports at most 49152 tiles");
  SelectArgs a{};
  a.g = G;
  a.qm = qm;
  a.km = km;
  a.scores = w.scores;
  a.Tld = w.Tld;
  a.keep = keep;
  a.mask = mask;
  a.near_tie = near_tie;
  a.qsplit = w.qsplit;
  a.ksplit = w.ksplit;
  a.gemm_ws = w.gemm_ws;
  a.gemm_ws_bytes = GEMM_WS_BYTES;
  for (int h0 = 0; h0 < G.H; h0 += w.hc) {
    a.h0 = h0;
    a.hc = G.H - h0 < w.hc ? G.H - h0 : w.hc;
    ZTRY(launch_scores(a, st));
    ZTRY(launch_select(a, st));
  }
  return ZEBRA_OK;
}

template <typename T>
static int run_sparse(const Geo& G, const void* q, const void* k, const void* v, long long ts, long long hs, int keep,
                      const uint32_t* mask_in, void* out, const SparseWs& w, bool norm_rope, float rope_base,
                      float eps, cudaStream_t st) {
  if (G.N == 0) return ZEBRA_OK;
  if (norm_rope) ZTRY(launch_rope_table(w.rope, nullptr, max_pos(G), (double)rope_base, st));
  PoolArgs<T> pa{};
  pa.g = G;
  pa.x[0] = static_cast<const T*>(q);
  pa.x[1] = static_cast<const T*>(k);
  pa.x[2] = static_cast<const T*>(v);
  pa.ts = ts;
  pa.hs = hs;
  pa.mean[0] = w.qm;
  pa.mean[1] = w.km;
  pa.mean[2] = w.vm;
  pa.packed[0] = static_cast<T*>(w.Qp);
  pa.packed[1] = static_cast<T*>(w.Kp);
  pa.packed[2] = static_cast<T*>(w.Vp);
  pa.lmk[0] = nullptr;
  pa.lmk[1] = static_cast<T*>(w.Kl);
  pa.lmk[2] = static_cast<T*>(w.Vl);
  pa.norm_rope[0] = pa.norm_rope[1] = norm_rope ? 1 : 0;
  pa.norm_rope[2] = 0;
  pa.rope = norm_rope ? w.rope : nullptr;
  pa.eps = eps;
  pa.counts = nullptr;
  pa.lmk_bias = w.lmk_bias;
  fill_ln_tab(pa.ln_tab);
  pa.dense_kv = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;   // the tcgen05 kernel's K/V layout
  if (G.T > 0) ZTRY(launch_pool_pack<T>(pa, 3, st));
  SpecialArgs<T> sa{};
  sa.g = G;
  sa.x[0] = pa.x[0];
  sa.x[1] = pa.x[1];
  sa.x[2] = pa.x[2];
  sa.ts = ts;
  sa.hs = hs;
  sa.out[0] = static_cast<T*>(w.Qs);
  sa.out[1] = static_cast<T*>(w.Ks);
  sa.out[2] = static_cast<T*>(w.Vs);
  sa.norm[0] = sa.norm[1] = norm_rope ? 1 : 0;
  sa.norm[2] = 0;
  sa.eps = eps;
  ZTRY(launch_pack_special<T>(sa, 3, st));
  const uint32_t* mask = mask_in;
  if (!mask && G.T > 0) {
    ZTRY(run_select(G, w.qm, w.km, keep, w.mask, nullptr, w.sel, st));
    mask = w.mask;
  }
  AttnArgs aa{};
  aa.g = G;
  aa.Qp = w.Qp; aa.Kp = w.Kp; aa.Vp = w.Vp;
  aa.Qs = w.Qs; aa.Ks = w.Ks; aa.Vs = w.Vs;
  aa.Kl = w.Kl; aa.Vl = w.Vl;
  aa.km = w.km; aa.vm = w.vm;
  aa.mask = mask;
  aa.keep = keep;
  aa.out = out;
  aa.part_o = w.part_o;
  aa.part_ml = w.part_ml;
  aa.splits = w.splits;
  aa.lmk_bias = w.lmk_bias;
  fill_ln_tab(aa.ln_tab);
  if (G.T > 0) ZTRY(launch_sparse_attn<T>(aa, st));
  ZTRY(launch_special_rows<T>(aa, st));
  return ZEBRA_OK;
}

template <typename T>
static int run_linear(const Geo& G, const void* q, const void* k, const void* v, long long ts, long long hs,
                      const float* A, const float* b, float rope_base, float eps, void* out, const LinearWs& w,
                      cudaStream_t st) {
  if (G.N == 0) return ZEBRA_OK;
  ZTRY(launch_rope_table(w.rope, w.rope_g, max_pos(G), (double)rope_base, st));
  LinearArgs a{};
  a.g = G;
  a.q = q; a.k = k; a.v = v;
  a.ts = ts; a.hs = hs;
  a.A = A; a.b = b;
  a.eps = eps;
  a.rope = w.rope;
  a.rope_g = w.rope_g;
  a.maxpos = max_pos(G);
  a.part = w.part;
  a.chunks = w.chunks;
  a.chunk_tokens = w.chunk_tokens;
  a.state = w.state;
  a.state_b = w.state_b;
  a.out = out;
  return launch_linear<T>(a, st);
}

}  // namespace zebra

using namespace zebra;

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

int32_t zebra_keep_count(double y, int32_t n_tiles) {
  if (!(y >= 0.0 && y < 1.0) || n_tiles < 1) return -1;
  return keep_of(y, n_tiles);
}

const char* zebra_last_error(void) { return g_err.c_str(); }
uint64_t zebra_launch_count(void) { return g_launches.load(); }
const char* zebra_version(void) { return "zebra-b200 0.1.0 (sm_100a)"; }

size_t zebra_workspace_bytes(const zebra_geom* g, int op, zebra_dtype dt, double y) {
  (void)y;
  if (check_geom(g) || check_dtype(dt)) return 0;
  const Geo G = make_geo(*g);
  Carver c(nullptr);
  switch (op) {
    case ZEBRA_OP_SELECT: {
      SelectWs w;
      carve_select(G, c, w);
      break;
    }
    case ZEBRA_OP_SPARSE: {
      SparseWs w;
      carve_sparse(G, dt, c, w);
      break;
    }
    case ZEBRA_OP_LINEAR: {
      LinearWs w;
      carve_linear(G, c, w);
      break;
    }
    case ZEBRA_OP_AFFINE:
      c.take<double>((size_t)G.H * affine_chunks(G) * AF_STRIDE);
      break;
    case ZEBRA_OP_HYBRID_LINEAR:
    case ZEBRA_OP_HYBRID_SPARSE:
    case ZEBRA_OP_HYBRID_DENSE: {
      HybridWs w;
      carve_hybrid(G, op == ZEBRA_OP_HYBRID_LINEAR ? ZEBRA_LAYER_LINEAR : ZEBRA_LAYER_SPARSE, c, w);
      break;
    }
    default:
      set_error("unknown op");
      return 0;
  }
  return c.used() ? c.used() : 256;
}

int zebra_tile_pool(const zebra_geom* g, zebra_dtype dt, const void* x, const zebra_layout* layout, float* x_mean,
                    void* x_packed, int32_t* tile_counts, void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_dtype(dt));
  long long ts, hs;
  ZTRY(check_layout(g, dt, layout, &ts, &hs));
  const Geo G = make_geo(*g);
  if (G.T == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(x, "x"));
  ZTRY(check_ptr16(x_mean, "x_mean"));
  if (x_packed) ZTRY(check_ptr16(x_packed, "x_packed"));
  ZTRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == ZEBRA_BF16) {
    PoolArgs<__nv_bfloat16> a{};
    a.g = G;
    a.x[0] = static_cast<const __nv_bfloat16*>(x);
    a.ts = ts;
    a.hs = hs;
    a.mean[0] = x_mean;
    a.packed[0] = static_cast<__nv_bfloat16*>(x_packed);
    a.counts = tile_counts;
    return launch_pool_pack(a, 1, st);
  }
  PoolArgs<float> a{};
  a.g = G;
  a.x[0] = static_cast<const float*>(x);
  a.ts = ts;
  a.hs = hs;
  a.mean[0] = x_mean;
  a.packed[0] = static_cast<float*>(x_packed);
  a.counts = tile_counts;
  return launch_pool_pack(a, 1, st);
}

int zebra_tile_select(const zebra_geom* g, const float* q_mean, const float* k_mean, double y, uint32_t* mask,
                      uint8_t* near_tie, int32_t* k_out, void* workspace, size_t ws_bytes, void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_y(y));
  const Geo G = make_geo(*g);
  if (G.T > SELECT_MAX_T) return fail(ZEBRA_ERR_UNSUPPORTED, "selection supports at most 49152 tiles");
  const int keep = G.T > 0 ? keep_of(y, G.T) : 0;
  if (k_out) *k_out = keep;
  if (G.T == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(q_mean, "q_mean"));
  ZTRY(check_ptr16(k_mean, "k_mean"));
  if (!mask) return fail(ZEBRA_ERR_INVALID_ARG, "mask is null");
  Carver c(workspace);
  SelectWs w;
  carve_select(G, c, w);
  ZTRY(check_workspace(workspace, ws_bytes, c.used()));
  ZTRY(check_device());
  return run_select(G, q_mean, k_mean, keep, mask, near_tie, w, static_cast<cudaStream_t>(stream));
}

int zebra_sparse_attn(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k, const void* v,
                      const zebra_layout* layout, double y, const uint32_t* mask, void* out, void* workspace,
                      size_t ws_bytes, void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_dtype(dt));
  ZTRY(check_y(y));
  long long ts, hs;
  ZTRY(check_layout(g, dt, layout, &ts, &hs));
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(q, "q"));
  ZTRY(check_ptr16(k, "k"));
  ZTRY(check_ptr16(v, "v"));
  ZTRY(check_ptr16(out, "out"));
  if (!mask && G.T > SELECT_MAX_T) return fail(ZEBRA_ERR_UNSUPPORTED, "selection supports at most 49152 tiles");
  if ((long long)G.T * G.H * 64 > 0x7fffffffLL)
    return fail(ZEBRA_ERR_UNSUPPORTED, "tiles x heads x 64 must stay below 2^31 (32-bit TMA row coordinates)");
  Carver c(workspace);
  SparseWs w;
  carve_sparse(G, dt, c, w);
  ZTRY(check_workspace(workspace, ws_bytes, c.used()));
  ZTRY(check_device());
  const int keep = G.T > 0 ? keep_of(y, G.T) : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == ZEBRA_BF16)
    return run_sparse<__nv_bfloat16>(G, q, k, v, ts, hs, keep, mask, out, w, false, 100.f, 1e-6f, st);
  return run_sparse<float>(G, q, k, v, ts, hs, keep, mask, out, w, false, 100.f, 1e-6f, st);
}

int zebra_linear_attn(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k, const void* v,
                      const zebra_layout* layout, const float* A, const float* b, float rope_base, float eps,
                      void* out, void* workspace, size_t ws_bytes, void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_dtype(dt));
  long long ts, hs;
  ZTRY(check_layout(g, dt, layout, &ts, &hs));
  if (!(rope_base > 0.f) || !(eps >= 0.f)) return fail(ZEBRA_ERR_INVALID_ARG, "rope_base must be > 0 and eps >= 0");
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(q, "q"));
  ZTRY(check_ptr16(k, "k"));
  ZTRY(check_ptr16(v, "v"));
  ZTRY(check_ptr16(out, "out"));
  Carver c(workspace);
  LinearWs w;
  carve_linear(G, c, w);
  ZTRY(check_workspace(workspace, ws_bytes, c.used()));
  ZTRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == ZEBRA_BF16) return run_linear<__nv_bfloat16>(G, q, k, v, ts, hs, A, b, rope_base, eps, out, w, st);
  return run_linear<float>(G, q, k, v, ts, hs, A, b, rope_base, eps, out, w, st);
}

int zebra_affine_moments(const zebra_geom* g, zebra_dtype dt, const void* x, const void* y,
                         const zebra_layout* layout, int per_head, double* moments, void* workspace, size_t ws_bytes,
                         void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_dtype(dt));
  long long ts, hs;
  ZTRY(check_layout(g, dt, layout, &ts, &hs));
  if (per_head != 0 && per_head != 1) return fail(ZEBRA_ERR_INVALID_ARG, "per_head must be 0 or 1");
  if (!moments || (reinterpret_cast<uintptr_t>(moments) & 7))
    return fail(ZEBRA_ERR_INVALID_ARG, "moments must be non-null and 8-byte aligned");
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(x, "x"));
  ZTRY(check_ptr16(y, "y"));
  AffineArgs a{};
  a.g = G;
  a.x = x;
  a.y = y;
  a.ts = ts;
  a.hs = hs;
  a.per_head = per_head;
  a.chunks = affine_chunks(G);
  a.chunk_tokens = (int)((G.N + a.chunks - 1) / a.chunks);
  a.moments = moments;
  Carver c(workspace);
  a.part = c.take<double>((size_t)G.H * a.chunks * AF_STRIDE);
  ZTRY(check_workspace(workspace, ws_bytes, c.used()));
  ZTRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == ZEBRA_BF16 ? launch_affine_moments<__nv_bfloat16>(a, st) : launch_affine_moments<float>(a, st);
}

int zebra_affine_solve(const zebra_geom* g, const double* moments, int per_head, double lam, float* A, float* b,
                       void* stream) {
  ZTRY(check_geom(g));
  if (per_head != 0 && per_head != 1) return fail(ZEBRA_ERR_INVALID_ARG, "per_head must be 0 or 1");
  if (!(lam >= 0.0) || !std::isfinite(lam)) return fail(ZEBRA_ERR_INVALID_ARG, "lam must be finite and >= 0");
  if (!moments || (reinterpret_cast<uintptr_t>(moments) & 7))
    return fail(ZEBRA_ERR_INVALID_ARG, "moments must be non-null and 8-byte aligned");
  if (!A || !b || (reinterpret_cast<uintptr_t>(A) & 3) || (reinterpret_cast<uintptr_t>(b) & 3))
    return fail(ZEBRA_ERR_INVALID_ARG, "A and b must be non-null and 4-byte aligned");
  ZTRY(check_device());
  return launch_affine_solve(moments, per_head, g->heads, lam, A, b, static_cast<cudaStream_t>(stream));
}

size_t zebra_coverage_workspace_bytes(const zebra_geom* g, int32_t n_query_tiles) {
  if (check_geom(g)) return 0;
  if (n_query_tiles < 1 || n_query_tiles > COV_MAX_TILES) {
    set_error("n_query_tiles must lie in [1, 1024]");
    return 0;
  }
  const Geo G = make_geo(*g);
  if (G.T == 0) return 256;
  return align256((size_t)n_query_tiles * G.H * coverage_splits(G, n_query_tiles) * 64 * sizeof(float4));
}

int zebra_coverage(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k, const zebra_layout* layout,
                   const uint32_t* mask, const int32_t* query_tiles, int32_t n_query_tiles, float* selected_mass,
                   float* special_mass, void* workspace, size_t ws_bytes, void* stream) {
  ZTRY(check_geom(g));
  ZTRY(check_dtype(dt));
  if (dt != ZEBRA_BF16) return fail(ZEBRA_ERR_UNSUPPORTED, "the coverage diagnostic takes bf16 Q and K");
  long long ts, hs;
  ZTRY(check_layout(g, dt, layout, &ts, &hs));
  const Geo G = make_geo(*g);
  if (n_query_tiles < 1 || n_query_tiles > COV_MAX_TILES)
    return fail(ZEBRA_ERR_INVALID_ARG, "n_query_tiles must lie in [1, 1024]");
  if (!query_tiles) return fail(ZEBRA_ERR_INVALID_ARG, "query_tiles is null");
  for (int32_t i = 0; i < n_query_tiles; ++i)
    if (query_tiles[i] < 0 || query_tiles[i] >= G.T)
      return fail(ZEBRA_ERR_INVALID_ARG, "query tile index outside [0, T)");
  ZTRY(check_ptr16(q, "q"));
  ZTRY(check_ptr16(k, "k"));
  if (!mask) return fail(ZEBRA_ERR_INVALID_ARG, "mask is null");
  if (!selected_mass || !special_mass) return fail(ZEBRA_ERR_INVALID_ARG, "output pointers are null");
  CoverageArgs a{};
  a.g = G;
  a.q = q;
  a.k = k;
  a.ts = ts;
  a.hs = hs;
  a.mask = mask;
  a.n = n_query_tiles;
  a.splits = coverage_splits(G, n_query_tiles);
  const size_t need = (size_t)a.n * G.H * a.splits * 64 * sizeof(float4);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15))
    return fail(ZEBRA_ERR_WORKSPACE, "workspace too small (zebra_coverage_workspace_bytes) or misaligned");
  a.part = static_cast<float4*>(workspace);
  a.sel = selected_mass;
  a.spec = special_mass;
  for (int32_t i = 0; i < n_query_tiles; ++i) a.tiles[i] = query_tiles[i];
  ZTRY(check_device());
  return launch_coverage(a, static_cast<cudaStream_t>(stream));
}

int zebra_affine_residual(const zebra_geom* g, const double* moments, int per_head, const float* A, const float* b,
                          double* err, void* stream) {
  ZTRY(check_geom(g));
  if (per_head != 0 && per_head != 1) return fail(ZEBRA_ERR_INVALID_ARG, "per_head must be 0 or 1");
  if (!moments || (reinterpret_cast<uintptr_t>(moments) & 7) || !err || (reinterpret_cast<uintptr_t>(err) & 7))
    return fail(ZEBRA_ERR_INVALID_ARG, "moments and err must be non-null and 8-byte aligned");
  if (!A || !b || (reinterpret_cast<uintptr_t>(A) & 3) || (reinterpret_cast<uintptr_t>(b) & 3))
    return fail(ZEBRA_ERR_INVALID_ARG, "A and b must be non-null and 4-byte aligned");
  ZTRY(check_device());
  return launch_affine_residual(moments, per_head, g->heads, A, b, err, static_cast<cudaStream_t>(stream));
}

int32_t zebra_allocate_layers(const double* errors, int32_t n_layers, double linear_fraction, int32_t* is_linear) {
  if (n_layers < 0 || !(linear_fraction >= 0.0 && linear_fraction <= 1.0)) return -1;
  if (n_layers > 0 && (!errors || !is_linear)) return -1;
  const int32_t count = (int32_t)floor(linear_fraction * (double)n_layers + 0.5);
  std::vector<int32_t> order((size_t)n_layers);
  for (int32_t i = 0; i < n_layers; ++i) order[(size_t)i] = i;
  // ascending error, NaN last, equal errors in index order
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t c) {
    const double ea = errors[a], ec = errors[c];
    if (std::isnan(ea)) return false;
    if (std::isnan(ec)) return true;
    return ea < ec;
  });
  for (int32_t i = 0; i < n_layers; ++i) is_linear[i] = 0;
  for (int32_t r = 0; r < count; ++r) is_linear[order[(size_t)r]] = 1;
  return count;
}

int zebra_hybrid_layer(const zebra_geom* g, int kind, const void* x, const void* w_qkv, const void* w_o,
                       const float* A, const float* b, double y, float rope_base, float eps, void* x_out,
                       void* workspace, size_t ws_bytes, void* stream) {
  ZTRY(check_geom(g));
  if (kind != ZEBRA_LAYER_LINEAR && kind != ZEBRA_LAYER_SPARSE && kind != ZEBRA_LAYER_DENSE)
    return fail(ZEBRA_ERR_INVALID_ARG, "unknown layer kind");
  if (kind == ZEBRA_LAYER_SPARSE) ZTRY(check_y(y));
  if (!(rope_base > 0.f) || !(eps >= 0.f)) return fail(ZEBRA_ERR_INVALID_ARG, "rope_base must be > 0 and eps >= 0");
  const Geo G = make_geo(*g);
  if (G.N == 0) return ZEBRA_OK;
  ZTRY(check_ptr16(x, "x"));
  ZTRY(check_ptr16(w_qkv, "w_qkv"));
  ZTRY(check_ptr16(w_o, "w_o"));
  ZTRY(check_ptr16(x_out, "x_out"));
  if (kind != ZEBRA_LAYER_LINEAR && G.T > SELECT_MAX_T)
    return fail(ZEBRA_ERR_UNSUPPORTED, "selection supports at most 49152 tiles");
  if (kind != ZEBRA_LAYER_LINEAR && (long long)G.T * G.H * 64 > 0x7fffffffLL)
    return fail(ZEBRA_ERR_UNSUPPORTED, "tiles x heads x 64 must stay below 2^31 (32-bit TMA row coordinates)");
  Carver c(workspace);
  HybridWs w;
  carve_hybrid(G, kind, c, w);
  ZTRY(check_workspace(workspace, ws_bytes, c.used()));
  ZTRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long Dm = (long long)G.H * D;
  ZTRY(gemm_bf16_nt(x, w_qkv, nullptr, w.qkv, G.N, 3 * Dm, Dm, 0.f, w.gemm_ws, GEMM_WS_BYTES, st));
  const __nv_bfloat16* qkv = static_cast<const __nv_bfloat16*>(w.qkv);
  const void* q = qkv;
  const void* k = qkv + Dm;
  const void* v = qkv + 2 * Dm;
  const long long ts = 3 * Dm, hs = D;
  if (kind == ZEBRA_LAYER_LINEAR) {
    ZTRY(run_linear<__nv_bfloat16>(G, q, k, v, ts, hs, A, b, rope_base, eps, w.o, w.li, st));
  } else {
    const int keep = kind == ZEBRA_LAYER_DENSE ? G.T : keep_of(y, G.T);
    ZTRY(run_sparse<__nv_bfloat16>(G, q, k, v, ts, hs, keep, nullptr, w.o, w.sp, true, rope_base, eps, st));
  }
  if (x_out != x) return gemm_bf16_nt(w.o, w_o, x, x_out, G.N, Dm, Dm, 1.f, w.gemm_ws, GEMM_WS_BYTES, st);
  // In place: a GEMM whose C and D alias may read C after writing D, so the
  // result goes to the QKV scratch (no longer needed) and is then copied over x.
  ZTRY(gemm_bf16_nt(w.o, w_o, x, w.qkv, G.N, Dm, Dm, 1.f, w.gemm_ws, GEMM_WS_BYTES, st));
  const cudaError_t e = cudaMemcpyAsync(x_out, w.qkv, (size_t)G.N * Dm * sizeof(__nv_bfloat16),
                                        cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return fail(ZEBRA_ERR_CUDA, std::string("in-place copy: ") + cudaGetErrorString(e));
  return ZEBRA_OK;
}

int zebra_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_recs.clear();
  g_prof_on.store(on != 0);
  if (on) {
    if (int rc = check_device()) return rc;
    reset_logit_counters();
    return check_launch("zebra_profile_enable");
  }
  return ZEBRA_OK;
}

long long zebra_profile_report(char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  struct Acc {
    long long records = 0, launches = 0;
    double ms = 0.0;
  };
  std::map<std::string, Acc> acc;
  std::vector<std::string> order;
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.a, r.b);
    if (acc.find(r.name) == acc.end()) order.push_back(r.name);
    Acc& x = acc[r.name];
    x.records += 1;
    x.launches += r.launches;
    x.ms += ms;
  }
  std::string out;
  char line[256];
  for (auto& n : order) {
    snprintf(line, sizeof(line), "kernel %s %lld %.6f %lld\n", n.c_str(), acc[n].records, acc[n].ms, acc[n].launches);
    out += line;
  }
  unsigned long long cnt[2] = {0, 0};
  if (check_device() == ZEBRA_OK) read_logit_counters(cnt);
  snprintf(line, sizeof(line), "logits sparse_rows %llu\nlogits special_rows %llu\n", cnt[0], cnt[1]);
  out += line;
  if (buf && len) {
    const size_t n = out.size() < len - 1 ? out.size() : len - 1;
    memcpy(buf, out.data(), n);
    buf[n] = 0;
  }
  return (long long)out.size();
}

int zebra_debug_inject(int32_t block, uint64_t wait_ns) {
  ZTRY(check_device());
  if (set_debug_inject(block, (unsigned long long)wait_ns) != ZEBRA_OK ||
      set_linear_debug_inject(block, (unsigned long long)wait_ns) != ZEBRA_OK)
    return fail(ZEBRA_ERR_CUDA, "setting the test hook failed");
  return ZEBRA_OK;
}

int zebra_sync_status(void* stream) {
  const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(ZEBRA_ERR_CUDA, cudaGetErrorString(e));
  int st = 0;
  if (read_and_clear_status(&st) != ZEBRA_OK) return fail(ZEBRA_ERR_CUDA, "reading the device status word failed");
  int st_lin = 0;
  if (read_and_clear_linear_status(&st_lin) != ZEBRA_OK)
    return fail(ZEBRA_ERR_CUDA, "reading the device status word failed");
  if (st || st_lin) return fail(ZEBRA_ERR_TIMEOUT, "a device-side wait gave up (kernel aborted; outputs are invalid)");
  if (read_and_clear_affine_status(&st) != ZEBRA_OK)
    return fail(ZEBRA_ERR_CUDA, "reading the device status word failed");
  if (st) return fail(ZEBRA_ERR_NUMERIC, "an affine fit met a system that is not positive definite (A, b are NaN)");
  return ZEBRA_OK;
}

}  // extern "C"
