// Kernel argument structs and launcher declarations (internal).
#pragma once

#include "common.cuh"

namespace zebra {

template <typename T>
struct PoolArgs {
  Geo g;
  const T* x[3];        // up to three [N, H, d] inputs (Q, K, V); null = skip
  long long ts, hs;     // token / head strides in elements (shared)
  float* mean[3];       // [H, T, d] fp32 or null
  T* packed[3];         // [H, T, 64, d] or null; K and V (z = 1, 2) in the dense layout when dense_kv
  int dense_kv;         // K/V rows at h * V * RPV + dense_tile_row (see common.cuh), zero-padded to 8
  T* lmk[3];            // [H, Tpad, d] landmark rows (mean rounded to T) or null
  int norm_rope[3];     // apply RMS norm (+ rotation when rope != null)
  const float2* rope;   // [maxpos, 16] cos/sin table or null
  float eps;
  int32_t* counts;      // [T] or null
  float* lmk_bias;      // [T] or null: ln(n_u) log2(e), the logit bias of tile u's landmark
  float ln_tab[TOK + 1];   // ln(m), m = 0..64, for lmk_bias
};

template <typename T>
struct SpecialArgs {
  Geo g;
  const T* x[3];
  long long ts, hs;
  T* out[3];            // [H, NSp, d]
  int norm[3];
  float eps;
};

template <typename T> int launch_pool_pack(const PoolArgs<T>& a, int ntensors, cudaStream_t st);
template <typename T> int launch_pack_special(const SpecialArgs<T>& a, int ntensors, cudaStream_t st);
// tab_g (optional): the same table as packed-pair operands of the linear kernels
int launch_rope_table(float2* tab, float4* tab_g, int maxpos, double base, cudaStream_t st);

// ---- selector ----
struct SelectArgs {
  Geo g;
  const float* qm;      // [H, T, d]
  const float* km;
  float* scores;        // [hc, T, Tld]
  int Tld;
  int h0, hc;           // head range of this pass
  int keep;
  uint32_t* mask;       // [H, T, W]
  uint8_t* near_tie;    // [H, T] or null
  void* qsplit;         // [hc, T, 384] bf16: the query means as bf16 parts (see scores_split_kernel)
  void* ksplit;         // [hc, T, 384] bf16: the key means, parts in the matching order
  void* gemm_ws;        // cuBLASLt workspace for the score GEMM
  size_t gemm_ws_bytes;
};
constexpr int SPLIT_K = 6 * 64;   // the score GEMM's K: six products of bf16 parts
int launch_scores(const SelectArgs& a, cudaStream_t st);
int launch_select(const SelectArgs& a, cudaStream_t st);
constexpr int SELECT_MAX_T = 49152;

// ---- attention ----
struct AttnArgs {
  Geo g;
  const void* Qp;  const void* Kp;  const void* Vp;   // [H, T, 64, d]
  const void* Qs;  const void* Ks;  const void* Vs;   // [H, NSp, d]
  const void* Kl;  const void* Vl;                    // [H, Tpad, d] landmark rows
  const float* km; const float* vm;                   // [H, T, d] fp32 means (own-tile landmark)
  const uint32_t* mask;                               // [H, T, W]
  int keep;
  void* out;                                          // [N, H, d]
  // split-KV partials of the dense special-token rows
  float* part_o;                                      // [splits, H, NSp, d]
  float* part_ml;                                     // [splits, H, NSp, 2] (max in log2 units, sum)
  int splits;
  float ln_tab[TOK + 1];                              // ln(m), m = 0..64 (ln_tab[0] unused)
  const float* lmk_bias;                              // [T] ln(n_u) log2(e) per tile (landmark logit bias)
};
template <typename T> int launch_sparse_attn(const AttnArgs& a, cudaStream_t st);
int launch_sparse_attn_tc(const AttnArgs& a, cudaStream_t st);
int launch_special_rows_tc(const AttnArgs& a, cudaStream_t st);
// sticky device status word of the kernels with bounded waits (per device)
int read_and_clear_status(int* out);
// error-path test hook of the tcgen05 sparse kernel (current device)
int set_debug_inject(int block, unsigned long long wait_ns);
template <typename T> int launch_special_rows(const AttnArgs& a, cudaStream_t st);

// ---- attention-concentration diagnostic ----
constexpr int COV_MAX_TILES = 1024;   // sampled query tiles per call (passed as kernel parameters)
struct CoverageArgs {
  Geo g;
  const void* q; const void* k;       // [N, H, d] bf16, strided
  long long ts, hs;
  const uint32_t* mask;               // [H, T, W] selection
  int n, splits;
  float4* part;                       // [n, H, splits, 64]: (max, total, selected, special), log2 units
  float* sel; float* spec;            // [n, H, 64]
  int32_t tiles[COV_MAX_TILES];
};
int coverage_splits(const Geo& g, int n);
int launch_coverage(const CoverageArgs& a, cudaStream_t st);

// ---- linear stage ----
struct LinearArgs {
  Geo g;
  const void* q; const void* k; const void* v;
  long long ts, hs;
  const float* A; const float* b;   // [H, d, d], [H, d] or null
  float eps;
  const float2* rope;               // [maxpos, 16]
  const float4* rope_g;             // [8 pair groups, maxpos] (launch_rope_table's tab_g)
  int maxpos;
  float* part;                      // [chunks, H, d, 65] partial (S | z)
  int chunks, chunk_tokens;
  float* state;                     // [H, d, 65] fp32  S' = S A^T | z
  void* state_b;                    // [H, 72, d] bf16 B operand (transposed) for the bf16 apply
  void* out;                        // [N, H, d]
};
template <typename T> int launch_linear(const LinearArgs& a, cudaStream_t st);
int linear_chunks(const Geo& g, int* chunk_tokens);
// sticky status word and error-path test hook of the bf16 linear state kernel (current device)
int read_and_clear_linear_status(int* out);
int set_linear_debug_inject(int block, unsigned long long wait_ns);

// ---- closed-form affine fit ----
constexpr int AF_D = 64;
// one group's float64 moments: count, sum x, sum y, sum x x^T, sum x y^T, sum |y|^2
constexpr int AF_N = 0, AF_SX = 1, AF_SY = AF_SX + AF_D, AF_SXX = AF_SY + AF_D, AF_SXY = AF_SXX + AF_D * AF_D;
constexpr int AF_SYY = AF_SXY + AF_D * AF_D;
constexpr int AF_STRIDE = AF_SYY + 1;   // 8322
struct AffineArgs {
  Geo g;
  const void* x; const void* y;     // [N, H, d] samples (linear output, teacher output)
  long long ts, hs;
  int chunks, chunk_tokens;         // token chunks per head
  int per_head;
  double* part;                     // [H, chunks, AF_STRIDE] partial moments
  double* moments;                  // [groups, AF_STRIDE], accumulated into
};
int affine_chunks(const Geo& g);
template <typename T> int launch_affine_moments(const AffineArgs& a, cudaStream_t st);
int launch_affine_solve(const double* moments, int per_head, int heads, double lam, float* A, float* b,
                        cudaStream_t st);
int read_and_clear_affine_status(int* out);
int launch_affine_residual(const double* moments, int per_head, int heads, const float* A, const float* b,
                           double* err, cudaStream_t st);

}  // namespace zebra
