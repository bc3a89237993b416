// Tile-sparse softmax attention on the 5th-generation tensor cores (tcgen05).
//
// Page "How Hybrid Attention Lets Feed-Forward 3D Models Scale to Many Views",
// section "Linear-centered stages plus tile-sparse stages": selected tiles keep
// full softmax interactions, omitted tiles become mean key/value landmarks,
// special-token keys stay visible and each patch query keeps its self key.
// Section "Speedup scales with the number of input views": keys and values are
// packed tile-major. Here K and V use a dense layout of 8-row groups (the
// tile's rows, zero rows up to a multiple of 8), and the kept tiles' groups are
// packed 8 to a 64-key block, so the 37 x 37 grids' 40- and 25-token edge
// tiles fill whole blocks instead of leaving masked columns.
//
// One CTA = one (query tile, head): a 64-row query block against the stream of
// 64-key blocks (packed kept tiles, landmark blocks, special-key blocks)
// described in attn.cu. The block count is known up front (a pre-pass over the
// selection row), so only the producer walks the stream. Warp roles:
//   warp 0      producer: TMA loads of Q once and of the K and V tile of every
//               block (one 64-row copy, or for a packed block one copy per run
//               of a tile's 8-row groups, each issued by its own lane) into
//               rings of STAGES 128-byte-swizzled 64x64 bf16 tiles (separate K
//               and V barriers: QK^T may start as soon as K has landed); right
//               after the K copy the whole warp writes the block's 64 logit
//               biases (log2 units: 0, ln(n_u) for landmarks, -inf for masked
//               columns) into one of STAGES + 1 bias slots, or only flags a
//               block of 64 real keys as bias-free;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into one of NSBUF TMEM
//               score buffers (tcgen05.mma M=64 N=64, K-major A/B), issued up
//               to NSBUF blocks ahead of O += P V (P from shared memory,
//               K-major; V MN-major). The whole warp runs the loop and waits;
//               one elected lane issues each group of MMAs and its commits
//               from a single asm block (a lane-0 branch with one MMA per
//               statement costs several times more issue cycles per MMA);
//   warps 2..5  softmax warpgroup, straight-line per block: tcgen05.ld of S
//               (16x256b: rows spread over quads as in the m16n8 accumulator),
//               scale + bias (packed f32x2 FMA), running max (3-input max),
//               exp2, bf16 P into shared memory (stmatrix), and O rescaling in
//               TMEM only when a row maximum grows by more than 2^8 (the stale
//               maximum is exact as long as both the sum and O use it).
// Row sums: the MMA warp also accumulates L += P x ones (N = 16) on the tensor
// cores, so the denominator adds exactly the bf16 P values that O adds and the
// softmax warps spend no instructions on it.
// TMEM: NSBUF score buffers of 64 columns, then O (128 or 256 columns); M=64
// accumulators occupy lanes 0-15, 32-47, 64-79, 96-111, i.e. 16 rows per
// softmax warp. L sits in the other half of each lane quarter (lane offset 16)
// of O's first 16 columns. Every mbarrier wait is bounded by the global timer; on expiry
// the CTA records ZEBRA_ERR_TIMEOUT in a device status word, drains its own
// copies and MMAs (bounded again), frees TMEM and exits.
// Included by attn.cu (one translation unit with the block iterator and the
// device counters).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tc_prims.cuh"

namespace zebra {

__device__ int g_status;   // sticky device status word (0 = ok)
// Error-path test hook (zebra_debug_inject): the limit of every bounded wait of
// the sparse kernel, and the block before which its producer stops issuing
// copies (-1 = never), so that a consumer's wait runs out.
__device__ unsigned long long g_wait_ns = 2000000000ull;
__device__ int g_inject_block = -1;

int set_debug_inject(int block, unsigned long long wait_ns) {
  const int b = block < 0 ? -1 : block;
  const unsigned long long w = wait_ns ? wait_ns : 2000000000ull;
  if (cudaMemcpyToSymbol(g_inject_block, &b, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_wait_ns, &w, sizeof(w)) != cudaSuccess)
    return ZEBRA_ERR_CUDA;
  return ZEBRA_OK;
}

int read_and_clear_status(int* out) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e != cudaSuccess) return ZEBRA_ERR_CUDA;
  const int z = 0;
  e = cudaMemcpyToSymbol(g_status, &z, sizeof(int));
  if (e != cudaSuccess) return ZEBRA_ERR_CUDA;
  *out = v;
  return ZEBRA_OK;
}

namespace tc {

#ifndef ZEBRA_TC_STAGES
#define ZEBRA_TC_STAGES 2
#endif
#ifndef ZEBRA_TC_CTAS
#define ZEBRA_TC_CTAS 4
#endif
constexpr int STAGES = ZEBRA_TC_STAGES;   // depth of the K and V rings
#ifndef ZEBRA_TC_NSBUF
#define ZEBRA_TC_NSBUF 1
#endif
constexpr int NSBUF = ZEBRA_TC_NSBUF;     // TMEM score buffers (QK^T lookahead)
#ifndef ZEBRA_TC_PBUF
#define ZEBRA_TC_PBUF 1
#endif
constexpr int PBUF = ZEBRA_TC_PBUF;       // shared-memory P buffers (softmax lead over PV)
constexpr int CTAS_PER_SM = ZEBRA_TC_CTAS;
#ifndef ZEBRA_TC_RSUM_MMA
#define ZEBRA_TC_RSUM_MMA 1
#endif
// 1: row sums as P x ones MMAs (N = 16) on the tensor cores; 0: in the softmax
// warps' registers (sums of the bf16-rounded exponentials: two more integer
// operations per pair, measured 3% slower than the MMAs)
constexpr bool RSUM_MMA = ZEBRA_TC_RSUM_MMA != 0;
#ifndef ZEBRA_TC_EMU
#define ZEBRA_TC_EMU 0
#endif
// of the 8 column groups a softmax thread holds per block, how many take
// their exponentials from the FMA-pipe polynomial (exp2_poly2) instead of the
// MUFU ex2 unit
constexpr int EMU = ZEBRA_TC_EMU;
static_assert(EMU >= 0 && EMU <= 8, "EMU counts column groups");
#ifndef ZEBRA_TC_PTMEM
#define ZEBRA_TC_PTMEM 0
#endif
// 1: the softmax writes P (bf16 pairs) into TMEM and O += P V reads its A
// operand from there. An M = 64 MMA with A in TMEM reads row m of A from the
// datapath lane that holds row m of its accumulator, so P and O share lanes
// 0-15 of each lane quarter (O in columns 0-63, two P buffers in 64-95 and
// 96-127), and the two score buffers of S = Q K^T use lanes 16-31 (columns 0-63
// and 64-127). The bias rows then live in a ring of 4 slots that the softmax
// releases, so S of block i + 2 never waits for O += P V of block i.
constexpr bool PTMEM = ZEBRA_TC_PTMEM != 0;
static_assert(!PTMEM || !RSUM_MMA, "P in TMEM keeps the row sums in registers");
constexpr int THREADS = 192;
// O (TMEM address offset): lanes 0-15 from column 0 (PTMEM) or after the
// first score buffer; a second score buffer without PTMEM uses lanes 16-31 of
// columns 0-63 (the row-sum accumulator L sits in lanes 16-31 of O's first 16)
constexpr uint32_t COL_O = PTMEM ? 0u : 64u;
constexpr uint32_t TMEM_COLS = PTMEM || COL_O + 64 <= 128 ? 128 : 256;
constexpr int PSM = PTMEM ? 0 : PBUF;    // shared-memory P buffers
// The bias rows go to a ring of 4 slots that the softmax releases when S runs
// two blocks ahead (PTMEM, or two score buffers): the producer then writes a
// block's row before it waits for a V stage, so S of block i + 2 never waits
// for O += P V of block i.
constexpr bool RING = PTMEM || NSBUF == 2;
#ifndef ZEBRA_TC_BIAS3
#define ZEBRA_TC_BIAS3 1
#endif
// Bias rows in STAGES + 1 slots, written right after the block's K copy: the
// slot of block i + 3 is free once QK^T of block i + 1 has completed (the
// producer has just waited for that to reuse the K stage), since that MMA
// was issued only after every softmax warp had signalled, after reading the
// row of block i, that it was done with block i's scores. Tied to the V stage
// instead, the row of block i waited for O += P V of block i - 2, and the MMA
// warp, which forwards the row to the softmax, waited with it.
constexpr bool BIAS3 = !RING && ZEBRA_TC_BIAS3 != 0;
constexpr int BST = RING ? 4 : (BIAS3 ? STAGES + 1 : STAGES);  // bias-row slots
#ifndef ZEBRA_TC_STAGGER
#define ZEBRA_TC_STAGGER 0
#endif
// nanoseconds by which the k-th CTA resident on an SM delays its first copy
// (k = its launch slot / SM count), to start the CTAs of an SM out of phase
constexpr int STAGGER_NS = ZEBRA_TC_STAGGER;
#ifndef ZEBRA_TC_KAHEAD
#define ZEBRA_TC_KAHEAD 0
#endif
// 1: the producer issues the K tile of block i + 1 before the V tile of block
// i, so a V stage still held by an unfinished O += P V no longer delays the
// next K tile (needs the bias ring of PTMEM)
constexpr bool KAHEAD = ZEBRA_TC_KAHEAD != 0;
static_assert(!KAHEAD || RING, "K ahead of V needs the bias-row ring");
// TMEM address offsets of score buffer b and (PTMEM) P buffer b
__host__ __device__ constexpr uint32_t s_addr(int b) { return PTMEM ? (16u << 16) + 64u * b : (uint32_t)b * (16u << 16); }
__host__ __device__ constexpr uint32_t p_addr_tmem(int b) { return 64u + 32u * b; }
constexpr uint32_t LANE_L = 16u << 16;   // TMEM lane offset of the row-sum accumulator L
constexpr unsigned long long DRAIN_NS = 200000000ull;   // 0.2 s while draining after an abort
static_assert(RING || NSBUF + 1 <= STAGES, "QK^T lookahead needs that many K stages");
static_assert(NSBUF <= 2 && PBUF <= 2, "at most two score and P buffers");

struct __align__(1024) Smem {
  __nv_bfloat16 q[64 * 64];
  __nv_bfloat16 k[STAGES][64 * 64];
  __nv_bfloat16 v[STAGES][64 * 64];
  __nv_bfloat16 p[PSM > 0 ? PSM : 1][PSM > 0 ? 64 * 64 : 8];
  __nv_bfloat16 ones[RSUM_MMA ? 16 * 64 : 8];  // B operand of the row-sum MMA (N = 16, K = 64), all 1.0
  float bias[BST][64];          // logit bias row of a block (log2 units)
  int all_zero[BST];            // 1 when every bias of the row is 0 (64 real keys, nothing masked)
  uint64_t q_full;
  uint64_t k_full[STAGES];
  uint64_t k_empty[STAGES];
  uint64_t v_full[STAGES];
  uint64_t v_empty[STAGES];
  uint64_t b_full[BST];         // bias row written
  uint64_t b_empty[BST];        // bias row read by the softmax (PTMEM)
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int nblocks;
  long long own_kv_row;         // packed: the own tile's first K/V row in the dense layout
};
// Shared memory per CTA: the layout, padded so that at most CTAS_PER_SM CTAs
// fit on an SM (their TMEM, CTAS_PER_SM x TMEM_COLS columns, must fit in 512).
constexpr size_t SMEM_NEED = sizeof(Smem) + 1024;
constexpr size_t SMEM_CAP = 227 * 1024;
constexpr size_t SMEM_FLOOR = SMEM_CAP / (CTAS_PER_SM + 1) + 1024;
constexpr size_t SMEM_BYTES = SMEM_NEED > SMEM_FLOOR ? SMEM_NEED : SMEM_FLOOR;
static_assert(SMEM_BYTES * CTAS_PER_SM <= SMEM_CAP, "shared memory layout");
static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "TMEM columns");

struct alignas(64) Params {
  // 64-row boxes; tkg / tvg: the dense K/V layout with boxes of 8 (m + 1) rows
  CUtensorMap tq, tkl, tvl, tks, tvs, tqs;
  CUtensorMap tkg[8], tvg[8];
  AttnArgs a;
  int item0;   // first work item of this launch; CTA b takes item0 + b
};

// Drain wait after an abort: waits for the phase whatever the abort flag says
// (copies or MMAs still in flight must land before the CTA frees its shared
// memory and TMEM), and gives up after `limit_ns`.
__device__ __noinline__ bool mbar_drain(uint64_t* b, uint32_t parity, unsigned long long limit_ns) {
  const unsigned long long t0 = gtime();
  while (!mbar_try(b, parity))
    if (gtime() - t0 > limit_ns) return false;
  return true;
}
__device__ __noinline__ bool mbar_drain_warp(uint64_t* b, uint32_t parity, unsigned long long limit_ns) {
  const unsigned long long t0 = gtime();
  while (true) {
    if (__all_sync(0xffffffffu, mbar_try(b, parity))) return true;
    if (__any_sync(0xffffffffu, gtime() - t0 > limit_ns)) return false;
  }
}

// Wait (all 32 lanes of a warp) for the phase of `parity` to complete; true
// when it did. The slow path keeps testing until the phase completes, another
// warp raises the abort flag, or the kernel's wait limit (g_wait_ns) passes;
// then it records the error status and raises the flag. The result is the
// same in every lane, so the loops around it stay converged for the elected
// issues below.
__device__ __noinline__ bool mbar_wait_warp_slow(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
  const unsigned long long limit_ns = *(volatile unsigned long long*)&g_wait_ns;
  const unsigned long long t0 = gtime();
  while (true) {
    if (__all_sync(0xffffffffu, mbar_try(b, parity))) return true;
    const bool late = gtime() - t0 > limit_ns;
    if (__any_sync(0xffffffffu, late || *abort_flag)) {
      if (late) {
        atomicExch(&g_status, ZEBRA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      __syncwarp();
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
  if (__all_sync(0xffffffffu, mbar_try(b, parity))) return true;
  return mbar_wait_warp_slow(b, parity, abort_flag);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(saddr(dst)), "l"(map), "r"(x), "r"(y), "r"(saddr(bar))
      : "memory");
}

// One elected lane of the (converged) warp arms `bar` with the tile's bytes and
// starts the copy.
__device__ __forceinline__ void tma_load_2d_elect(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%4], %5;\n"
      " @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n}\n"
      ::"r"(saddr(dst)), "l"(map), "r"(x), "r"(y), "r"(saddr(bar)), "r"(64 * 64 * 2)
      : "memory");
}

// One packed 64-row stage from the dense K/V layout: lane p copies piece p of
// the block (p_ng consecutive 8-row groups from row p_src, through the map
// whose box is 8 p_ng rows) to groups p_slot.. of the stage; lanes without a
// piece have p_ng = 0. The pieces, a zero-filled tail piece included (rows
// wholly outside the tensor), always cover the 8 groups, so lane 0 arms `bar`
// with the stage's full 8 KB before any copy starts. Every piece lands on a
// 1024-byte boundary, so the 128-byte swizzle gives the same layout as one
// 64-row copy.
__device__ __forceinline__ void tma_load_pieces(void* dst, const CUtensorMap* maps, int p_src, int p_slot, int p_ng,
                                                uint64_t* bar, int lane) {
  // one piece of all 8 groups (a whole 64-row tile): lane 0 arms and copies
  if (__shfl_sync(0xffffffffu, p_ng, 0) == 8) {
    if (lane == 0) {
      mbar_expect_tx(bar, 64 * 64 * 2);
      tma_load_2d(dst, maps + 7, 0, p_src, bar);
    }
    __syncwarp();
    return;
  }
  if (lane == 0) mbar_expect_tx(bar, 64 * 64 * 2);
  __syncwarp();
  if (p_ng > 0) tma_load_2d(static_cast<unsigned char*>(dst) + p_slot * 1024, maps + (p_ng - 1), 0, p_src, bar);
  __syncwarp();
}

// 8-row groups of tile u in the dense K/V layout
__device__ __forceinline__ int tile_groups(const Geo& g, int u) {
  const TileShape s = tile_shape(g, u);
  return (s.rows * s.cols + 7) >> 3;
}

// S = Q K^T (K = 64: four K = 16 steps) issued by one elected lane of the
// converged warp, then commits to `bar0` and `bar1`. One asm block keeps the
// issue cost per MMA low.
__device__ __forceinline__ void mma_qk_elect(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint64_t* bar0,
                                             uint64_t* bar1) {
  asm volatile(
      "{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, 0, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %9, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %9, p1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%10];\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%11];\n}\n"
      ::"r"(d), "l"(a), "l"(b), "l"(a + 2), "l"(b + 2), "l"(a + 4), "l"(b + 4), "l"(a + 6), "l"(b + 6), "r"(id),
      "r"(saddr(bar0)), "r"(saddr(bar1))
      : "memory");
}
// O += P V (V MN-major: K steps 2048 bytes apart) and L += P ones, then commits
// to `bar0` and `bar1`; `acc` = 0 starts both accumulators.
__device__ __forceinline__ void mma_pv_elect(uint32_t d_o, uint32_t d_l, uint64_t p, uint64_t v, uint64_t ones,
                                             uint32_t id_pv, uint32_t id_sum, uint32_t acc, uint64_t* bar0,
                                             uint64_t* bar1) {
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
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%17];\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%18];\n}\n"
      ::"r"(d_o), "r"(d_l), "l"(p), "l"(p + 2), "l"(p + 4), "l"(p + 6), "l"(v), "l"(v + 128), "l"(v + 256),
      "l"(v + 384), "l"(ones), "l"(ones + 2), "l"(ones + 4), "l"(ones + 6), "r"(id_pv), "r"(id_sum), "r"(acc),
      "r"(saddr(bar0)), "r"(saddr(bar1))
      : "memory");
}
// O += P V alone (row sums kept in the softmax warps' registers), then commits
// to `bar0` and `bar1`.
__device__ __forceinline__ void mma_pv_only_elect(uint32_t d_o, uint64_t p, uint64_t v, uint32_t id_pv, uint32_t acc,
                                                  uint64_t* bar0, uint64_t* bar1) {
  asm volatile(
      "{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, %10, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, p1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%11];\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%12];\n}\n"
      ::"r"(d_o), "l"(p), "l"(p + 2), "l"(p + 4), "l"(p + 6), "l"(v), "l"(v + 128), "l"(v + 256), "l"(v + 384),
      "r"(id_pv), "r"(acc), "r"(saddr(bar0)), "r"(saddr(bar1))
      : "memory");
}

// O += P V with P (the A operand, K-major bf16 pairs) in TMEM at `a_tmem`
// (8 columns per K = 16 step), V MN-major in shared memory; then commits to
// `bar0` and `bar1`.
__device__ __forceinline__ void mma_pv_tmem_elect(uint32_t d_o, uint32_t a_tmem, uint64_t v, uint32_t id_pv,
                                                  uint32_t acc, uint64_t* bar0, uint64_t* bar1) {
  asm volatile(
      "{\n .reg .pred e, p0, p1;\n setp.ne.b32 p0, %10, 0;\n setp.eq.b32 p1, 0, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %9, p0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %9, p1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %9, p1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%11];\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%12];\n}\n"
      ::"r"(d_o), "r"(a_tmem), "r"(a_tmem + 8), "r"(a_tmem + 16), "r"(a_tmem + 24), "l"(v), "l"(v + 128),
      "l"(v + 256), "l"(v + 384), "r"(id_pv), "r"(acc), "r"(saddr(bar0)), "r"(saddr(bar1))
      : "memory");
}

// P of one block (bf16 pairs, this thread's rows g4 and g4 + 8 of its warp's
// 16, pair j at column 4 j + q4) into TMEM at `taddr` (32 columns)
__device__ __forceinline__ void tmem_st_p(uint32_t taddr, const uint32_t (&pk)[8][2]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(pk[0][0]), "r"(pk[0][1]), "r"(pk[1][0]), "r"(pk[1][1]), "r"(pk[2][0]), "r"(pk[2][1]), "r"(pk[3][0]),
      "r"(pk[3][1]), "r"(pk[4][0]), "r"(pk[4][1]), "r"(pk[5][0]), "r"(pk[5][1]), "r"(pk[6][0]), "r"(pk[6][1]),
      "r"(pk[7][0]), "r"(pk[7][1])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 TMEM lanes x 64 fp32 columns -> 32 registers (m16n8 accumulator layout per 8 columns)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* r) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
        "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
        "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float* r) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(r);
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
      "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15]), "r"(u[16]), "r"(u[17]),
      "r"(u[18]), "r"(u[19]), "r"(u[20]), "r"(u[21]), "r"(u[22]), "r"(u[23]), "r"(u[24]), "r"(u[25]), "r"(u[26]),
      "r"(u[27]), "r"(u[28]), "r"(u[29]), "r"(u[30]), "r"(u[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* r) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(r);
  asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(u[0]), "r"(u[1]),
               "r"(u[2]), "r"(u[3])
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// (a.x, a.y) * (b.x, b.y) + (c.x, c.y) as one packed fp32 instruction
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2,%3};\n mov.b64 rb, {%4,%5};\n mov.b64 rc, {%6,%7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0,%1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair (x <= 8) on the FMA pipe: clamp to >= -126, x = j + f with
// j = round-to-nearest(x) (adding 1.5 * 2^23 leaves j in the low mantissa
// bits), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial minimax in relative
// error on that interval (coefficients from linear_global_attention_b200/
// exp2_fit.py, max relative error 7.5e-5); 2^j enters by an integer add to the
// exponent field.
constexpr float EXP2_C0 = 0.9999280571937561f, EXP2_C1 = 0.6932608485221863f, EXP2_C2 = 0.24261115491390228f,
                EXP2_C3 = 0.05517221987247467f;
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 one = make_float2(1.f, 1.f), mone = make_float2(-1.f, -1.f);
  const float2 magic = make_float2(12582912.f, 12582912.f), nmagic = make_float2(-12582912.f, -12582912.f);
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = ffma2(x, one, magic);      // 1.5 * 2^23 + j
  const float2 j = ffma2(t, one, nmagic);     // j (exact)
  const float2 f = ffma2(j, mone, x);         // x - j (exact)
  float2 p = ffma2(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  p = ffma2(p, f, make_float2(EXP2_C1, EXP2_C1));
  p = ffma2(p, f, make_float2(EXP2_C0, EXP2_C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// maximum of one row's 16 values in the 16x256b fragment (sv[4j + O], sv[4j + O + 1], j < 8),
// as a tree of 3-input maxima
template <int O>
__device__ __forceinline__ float max_row(const float* sv) {
  const float a = fmax3(sv[O + 0], sv[O + 1], sv[O + 4]), b = fmax3(sv[O + 5], sv[O + 8], sv[O + 9]);
  const float c = fmax3(sv[O + 12], sv[O + 13], sv[O + 16]), d = fmax3(sv[O + 17], sv[O + 20], sv[O + 21]);
  const float e = fmax3(sv[O + 24], sv[O + 25], sv[O + 28]);
  return fmaxf(fmax3(a, b, c), fmax3(d, e, sv[O + 29]));
}

// four 8x8 bf16 matrices from mma-fragment registers to shared memory; this
// thread gives the row address of row (lane & 7) of matrix (lane >> 3)
__device__ __forceinline__ void stmatrix4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}

// rows of block `id` of `kind` in the 2D [rows, 64] tensor map of its source
__device__ __forceinline__ int block_row(const Geo& g, int h, int kind, int id) {
  if (kind == 0) return (h * g.T + id) * 64;
  if (kind == 1) return h * g.Tpad + id * 64;
  return h * g.NSp + id * 64;
}

// MODE 0: patch query rows of the tile-sparse stage; work item h * T + t.
// MODE 1: dense special-token query rows: work item (h * splits + sp) * NQB + qb
// is query block qb (64 special queries, packed) of head h against key split
// sp (the key tiles [T sp / splits, T (sp + 1) / splits), plus every special
// key in split 0); it writes the split's unnormalised output, row maximum and
// row sum for special_combine_kernel.
// PACK: the grid has partial tiles, so kept tiles are packed 8 groups to a
// block; without partial tiles every tile is one whole block (the dense layout
// then coincides with 64-row tiles) and the packing code is compiled out.
template <int MODE, bool PACK>
__global__ void __launch_bounds__(THREADS, CTAS_PER_SM) attn_tc_kernel(const __grid_constant__ Params P) {
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnArgs& a = P.a;
  const Geo& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = P.item0 + (int)blockIdx.x;
  int h, t = 0, qb = 0, sp = 0, u0 = 0, u1 = 0;
  if constexpr (MODE == 0) {
    h = item / g.T;
    t = item - h * g.T;
  } else {
    const int nqb = g.NSp / 64;
    qb = item % nqb;
    const int hsp = item / nqb;
    sp = hsp % a.splits;
    h = hsp / a.splits;
    u0 = (int)((long long)g.T * sp / a.splits);
    u1 = (int)((long long)g.T * (sp + 1) / a.splits);
  }
  const uint32_t* mrow = MODE == 0 ? a.mask + ((size_t)h * g.T + t) * g.W : nullptr;
  volatile int* abort_flag = &sm.abort;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < BST; ++s) {
      mbar_init(&sm.b_full[s], 1);
      mbar_init(&sm.b_empty[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 2);   // MMA completion + the MMA thread's release after the bias row
      mbar_init(&sm.s_free[b], 4);
      mbar_init(&sm.p_full[b], 4);
      mbar_init(&sm.pv_done[b], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    if (MODE == 0 && PACK) sm.own_kv_row = (long long)h * g.V * g.RPV + dense_tile_row(g, t);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the all-ones operand of the row-sum MMA (read by the tensor cores: async proxy)
  if (RSUM_MMA)
    for (int i = tid; i < 16 * 64 / 2; i += THREADS) reinterpret_cast<uint32_t*>(sm.ones)[i] = 0x3F803F80u;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 0) {
    if constexpr (MODE == 0) {
      // pre-pass, lane-parallel: the number of blocks the walk below will
      // produce (packed blocks of 8 groups of the kept tiles' rows, landmark
      // blocks with a visible landmark, special blocks)
      int ng = 0, nl = 0;
      for (int w = lane; w < g.W; w += 32) {
        uint32_t m = mask_word(mrow, w, g.T);
        if constexpr (PACK) {
          while (m) {
            const int b = __ffs(m) - 1;
            m &= m - 1;
            ng += tile_groups(g, w * 32 + b);
          }
        } else {
          ng += 8 * __popc(m);
        }
      }
      for (int lb = lane; lb < g.Tpad / 64; lb += 32) {
        int nvis;
        nl += lmk_visible(mrow, g, t, lb, nvis) != 0u ? 1 : 0;
      }
      ng = __reduce_add_sync(0xffffffffu, ng);
      nl = __reduce_add_sync(0xffffffffu, nl);
      if (lane == 0) sm.nblocks = (ng + 7) / 8 + nl + g.NSp / 64;
    } else {
      int ng = 0;
      if constexpr (PACK) {
        for (int u = u0 + lane; u < u1; u += 32) ng += tile_groups(g, u);
        ng = __reduce_add_sync(0xffffffffu, ng);
      } else {
        ng = 8 * (u1 - u0);
      }
      if (lane == 0) sm.nblocks = (ng + 7) / 8 + (sp == 0 ? g.NSp / 64 : 0);
    }
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sm.tmem_base)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nb = sm.nblocks;

  // MODE 0: the query tile's shape and whether it keeps its own tile;
  // MODE 1: n_t = the valid special queries of the block
  const bool own_kept = MODE == 0 ? ((__ldg(mrow + (t >> 5)) >> (t & 31)) & 1u) != 0 : true;
  const TileShape ts = tile_shape(g, t);
  const int n_t = MODE == 0 ? ts.rows * ts.cols : min(64, g.NS - qb * 64);

  if (warp == 0) {
    // ---------------- producer (whole warp; one elected lane issues) ----------------
    int issued = 0, nk = 0, nvv = 0;   // blocks taken from the stream; K and V copies issued
    const int inject = *(volatile int*)&g_inject_block;   // error-path test hook (-1: off)
    if (STAGGER_NS > 0) __nanosleep((unsigned)(STAGGER_NS * (((int)blockIdx.x / 148) & 3)));
    BlockIter it{};
    if constexpr (MODE == 0) {
      tma_load_2d_elect(sm.q, &P.tq, 0, (h * g.T + t) * 64, &sm.q_full);
      iter_init(it, mrow, g);
    } else {
      tma_load_2d_elect(sm.q, &P.tqs, 0, h * g.NSp + qb * 64, &sm.q_full);
      it.w = u0;
      it.t_end = u1;
    }
    int kind, id, nv;
    long long keys = 0;   // visible keys per query row (for the logit counter)
    bool ok = true;
    // Key tiles (kind 0) are packed: their rows, in walk order and in the
    // dense layout's 8-row groups (real rows, then zero rows up to a multiple
    // of 8), fill the blocks 8 groups at a time, so an edge tile of 40 rows
    // and a corner tile of 25 share blocks with the next tiles instead of
    // leaving 24 or 39 masked columns each. For the current block, lane j < 8
    // holds the count of real rows of group j (gcnt), and lane p the p-th
    // piece (a run of groups of one tile, or the zero-filled tail): its source
    // row, first group and group count (p_src, p_slot, p_ng).
    // cur_row: the current tile's next group (its source row), cur_left: the
    // tile's real rows from there on (<= 0 once it is used up)
    int cur_row = 0, cur_left = 0;
    bool tiles_done = false;
    int gcnt = 0, p_src = 0, p_slot = 0, p_ng = 0;
    auto next_block = [&](int& bk, int& bid, int& bnv) -> bool {
      if (PACK && !tiles_done) {
        int slot = 0, np = 0;
        gcnt = 0;
        p_ng = 0;
        while (slot < 8) {
          if (cur_left <= 0) {
            // the next kept tile (MODE 1: the next tile of the key split)
            int u;
            bool more;
            if constexpr (MODE == 0) {
              while (it.bits == 0 && it.w + 1 < g.W) {
                ++it.w;
                it.bits = it.nxt;
                it.nxt = it.w + 1 < g.W ? mask_word(mrow, it.w + 1, g.T) : 0u;
              }
              more = it.bits != 0;
              u = it.w * 32 + __ffs(it.bits) - 1;
              it.bits &= it.bits - 1;
            } else {
              more = it.w < it.t_end;
              u = it.w++;
            }
            if (!more) {
              // the tiles are done: the walk goes on with the landmark
              // (MODE 0) or special blocks
              tiles_done = true;
              it.phase = MODE == 0 ? 1 : 2;
              break;
            }
            const TileShape sh = tile_shape(g, u);
            cur_row = h * g.V * g.RPV + sh.view * g.RPV + TILE * g.Wp * (sh.r0 / TILE) + sh.rows * sh.c0;
            cur_left = sh.rows * sh.cols;
            keys += cur_left;
          }
          const int take = min(8 - slot, (cur_left + 7) >> 3);
          const int j = lane - slot;
          if (j >= 0 && j < take) gcnt = min(8, cur_left - 8 * j);
          if (lane == np) {
            p_src = cur_row;
            p_slot = slot;
            p_ng = take;
          }
          ++np;
          slot += take;
          cur_row += 8 * take;
          cur_left -= 8 * take;
        }
        if (slot > 0) {
          if (slot < 8 && lane == np) {   // zero-filled tail: rows wholly before the tensor
            p_src = -64;
            p_slot = slot;
            p_ng = 8 - slot;
          }
          bk = 0;
          bid = 0;
          bnv = 0;   // the packed tiles' keys were counted as they were fetched
          return true;
        }
      }
      const bool more = MODE == 0 ? next_block_sparse(it, g, mrow, t, true, bk, bid, bnv)
                                  : next_block_dense(it, g, sp == 0, bk, bid, bnv);
      return more;
    };
    // V copy of block nvv (its stage's release is that of O += P V of block nvv - STAGES)
    auto issue_v = [&](int vkind, int vrow, int vsrc, int vslot, int vng) -> bool {
      const int vs = nvv % STAGES;
      if (nvv >= STAGES && !mbar_wait_warp(&sm.v_empty[vs], ((nvv / STAGES) - 1) & 1, abort_flag)) return false;
      if (PACK && vkind == 0)
        tma_load_pieces(sm.v[vs], P.tvg, vsrc, vslot, vng, &sm.v_full[vs], lane);
      else
        tma_load_2d_elect(sm.v[vs], vkind == 0 ? &P.tvg[7] : vkind == 1 ? &P.tvl : &P.tvs, 0, vrow, &sm.v_full[vs]);
      ++nvv;
      return true;
    };
    // KAHEAD: the block whose V copy is still to be issued
    int pend_kind = -1, pend_row = 0, pend_src = 0, pend_slot = 0, pend_ng = 0;
    while (ok && next_block(kind, id, nv)) {
      // test hook: stop before this block, so the MMA warp's wait for its K tile runs out
      if (issued == inject) break;
      keys += nv;
      const int s = issued % STAGES;
      const uint32_t par = ((issued / STAGES) - 1) & 1;
      // without packing a kept tile's rows start at (h T + id) 64, as in 64-row tiles
      const int row = kind == 0 && PACK ? 0 : block_row(g, h, kind, id);
      if (issued >= STAGES) ok = mbar_wait_warp(&sm.k_empty[s], par, abort_flag);
      if (!ok) break;
      if (PACK && kind == 0)
        tma_load_pieces(sm.k[s], P.tkg, p_src, p_slot, p_ng, &sm.k_full[s], lane);
      else
        tma_load_2d_elect(sm.k[s], kind == 0 ? &P.tkg[7] : kind == 1 ? &P.tkl : &P.tks, 0, row, &sm.k_full[s]);
      ++nk;
      // bias row of the block, two columns per lane, into slot issued % BST
      auto write_bias = [&]() {
        const int bs = issued % BST;
        float b0, b1;
        if (kind == 1) {
          b0 = block_bias(a, mrow, t, kind, id, 2 * lane);
          b1 = block_bias(a, mrow, t, kind, id, 2 * lane + 1);
        } else if (PACK && kind == 0) {
          // a block of 64 real keys needs no row: the softmax skips the bias
          if (__all_sync(0xffffffffu, lane >= 8 || gcnt == 8)) {
            if (lane == 0) {
              sm.all_zero[bs] = 1;
              mbar_arrive(&sm.b_full[bs]);
            }
            return;
          }
          // columns 2 lane, 2 lane + 1 sit in group lane / 4 at rows (2 lane) % 8, + 1
          const int vc = __shfl_sync(0xffffffffu, gcnt, lane >> 2);
          const int c0 = (2 * lane) & 7;
          b0 = c0 < vc ? 0.f : -INFINITY;
          b1 = c0 + 1 < vc ? 0.f : -INFINITY;
        } else {
          b0 = 2 * lane < nv ? 0.f : -INFINITY;
          b1 = 2 * lane + 1 < nv ? 0.f : -INFINITY;
        }
        *reinterpret_cast<float2*>(&sm.bias[bs][2 * lane]) = make_float2(b0, b1);
        const int zero = __all_sync(0xffffffffu, b0 == 0.f && b1 == 0.f);
        __threadfence_block();   // every lane's row entries precede lane 0's release below
        __syncwarp();
        if (lane == 0) {
          sm.all_zero[bs] = zero;
          mbar_arrive(&sm.b_full[bs]);
        }
      };
      if constexpr (RING) {
        // the slot is free once the softmax has read the row of block issued - BST
        if (issued >= BST) ok = mbar_wait_warp(&sm.b_empty[issued % BST], ((issued / BST) - 1) & 1, abort_flag);
        if (!ok) break;
        write_bias();
      }
      if constexpr (BIAS3) write_bias();
      // the V tile (and without PTMEM the bias row) of this stage is free once
      // PV of block issued - STAGES is done
      if constexpr (KAHEAD) {
        if (pend_kind >= 0) ok = issue_v(pend_kind, pend_row, pend_src, pend_slot, pend_ng);
        if (!ok) break;
        pend_kind = kind;
        pend_row = row;
        pend_src = p_src;
        pend_slot = p_slot;
        pend_ng = p_ng;
      } else {
        ok = issue_v(kind, row, p_src, p_slot, p_ng);
        if (!ok) break;
      }
      if constexpr (!RING && !BIAS3) write_bias();
      ++issued;
    }
    if (KAHEAD && ok && pend_kind >= 0)
      ok = issue_v(pend_kind, pend_row, pend_src, pend_slot, pend_ng);   // V of the last block
    if (lane == 0 && ok && issued == nb) {
      const long long extra = own_kept ? 0 : (n_t > 1 ? 2 : 1);   // the own-tile extras of the epilogue
      atomicAdd(&g_logits[MODE], (unsigned long long)((long long)n_t * (keys + extra)));
    }
    if (lane == 0 && (issued < nb || nvv < nb || *abort_flag)) {
      // stopped early: let the copies already in flight land before the CTA
      // frees its shared memory (the last STAGES copies into each ring are the
      // only ones whose landing nobody may have waited for)
      mbar_drain(&sm.q_full, 0, DRAIN_NS);
      for (int i = nk > STAGES ? nk - STAGES : 0; i < nk; ++i)
        mbar_drain(&sm.k_full[i % STAGES], (i / STAGES) & 1, DRAIN_NS);
      for (int i = nvv > STAGES ? nvv - STAGES : 0; i < nvv; ++i)
        mbar_drain(&sm.v_full[i % STAGES], (i / STAGES) & 1, DRAIN_NS);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    const uint32_t id_qk = idesc(false), id_pv = idesc(true), id_sum = idesc(false, 16);
    const uint64_t dq = desc_k(saddr(sm.q));
    const uint64_t d1 = desc_k(saddr(sm.ones));
    bool ok = mbar_wait_warp(&sm.q_full, 0, abort_flag);
    if constexpr (PTMEM) {
      // S = Q K^T of block q into score buffer q & 1 (free once the softmax
      // has loaded S of block q - 2), then the bias forward
      auto issue_qk = [&](int q) -> bool {
        const int s = q % STAGES, b = q & 1;
        if (!mbar_wait_warp(&sm.k_full[s], (q / STAGES) & 1, abort_flag)) return false;
        if (q >= 2 && !mbar_wait_warp(&sm.s_free[b], ((q >> 1) - 1) & 1, abort_flag)) return false;
        fence_after();
        mma_qk_elect(tmem + s_addr(b), dq, desc_k(saddr(sm.k[s])), id_qk, &sm.k_empty[s], &sm.s_full[b]);
        if (!mbar_wait_warp(&sm.b_full[q % BST], (q / BST) & 1, abort_flag)) return false;
        if (lane == 0) mbar_arrive(&sm.s_full[b]);
        __syncwarp();
        return true;
      };
      if (ok && nb > 0) ok = issue_qk(0);
      if (ok && nb > 1) ok = issue_qk(1);
      for (int j = 0; ok && j < nb; ++j) {
        if (j + 2 < nb) ok = issue_qk(j + 2);
        if (!ok) break;
        const int s = j % STAGES, b = j & 1;
        ok = mbar_wait_warp(&sm.v_full[s], (j / STAGES) & 1, abort_flag);
        if (ok) ok = mbar_wait_warp(&sm.p_full[b], (j >> 1) & 1, abort_flag);
        if (!ok) break;
        fence_after();
        // O += P V, P (the A operand) from P buffer b in the accumulator's lanes
        mma_pv_tmem_elect(tmem + COL_O, tmem + p_addr_tmem(b), desc_mn(saddr(sm.v[s])), id_pv, j > 0 ? 1u : 0u,
                          &sm.v_empty[s], &sm.pv_done[b]);
      }
    }
    int qk = 0;
    for (int j = 0; !PTMEM && ok && j < nb; ++j) {
      // S = Q K^T up to NSBUF blocks ahead of this PV (a score buffer is
      // reusable as soon as the softmax has loaded it)
      while (qk < nb && qk <= j + NSBUF) {
        const int s = qk % STAGES, b = qk % NSBUF;
        ok = mbar_wait_warp(&sm.k_full[s], (qk / STAGES) & 1, abort_flag);
        if (ok && qk >= NSBUF) ok = mbar_wait_warp(&sm.s_free[b], ((qk / NSBUF) - 1) & 1, abort_flag);
        if (!ok) break;
        fence_after();
        mma_qk_elect(tmem + s_addr(b), dq, desc_k(saddr(sm.k[s])), id_qk, &sm.k_empty[s], &sm.s_full[b]);
        // forward the stage's bias row to the softmax through s_full: this
        // warp acquires it here and releases it with one arrival
        ok = mbar_wait_warp(&sm.b_full[qk % BST], (qk / BST) & 1, abort_flag);
        if (!ok) break;
        if (lane == 0) mbar_arrive(&sm.s_full[b]);
        __syncwarp();
        ++qk;
      }
      if (!ok) break;
      // O += P V and L += P ones of block j
      const int s = j % STAGES, pb = j % PBUF;
      ok = mbar_wait_warp(&sm.v_full[s], (j / STAGES) & 1, abort_flag);
      if (ok) ok = mbar_wait_warp(&sm.p_full[pb], (j / PBUF) & 1, abort_flag);
      if (!ok) break;
      fence_after();
      if (RSUM_MMA)
        mma_pv_elect(tmem + COL_O, tmem + LANE_L + COL_O, desc_k(saddr(sm.p[pb])), desc_mn(saddr(sm.v[s])), d1,
                     id_pv, id_sum, j > 0 ? 1u : 0u, &sm.v_empty[s], &sm.pv_done[pb]);
      else
        mma_pv_only_elect(tmem + COL_O, desc_k(saddr(sm.p[pb])), desc_mn(saddr(sm.v[s])), id_pv, j > 0 ? 1u : 0u,
                          &sm.v_empty[s], &sm.pv_done[pb]);
    }
    // drain: every MMA this warp issued completes before TMEM is freed
    if (elect_one()) mma_commit(&sm.drain);
    __syncwarp();
    {
      const unsigned long long lim = *(volatile unsigned long long*)&g_wait_ns;
      mbar_drain_warp(&sm.drain, 0, *abort_flag ? DRAIN_NS + 0ull : lim);
    }
  } else {
    // ---------------- softmax warpgroup ----------------
    const int rb = warp & 3;                  // TMEM lane quarter this warp may access
    const int g4 = lane >> 2, q4 = lane & 3;
    const uint32_t lane_off = (uint32_t)(32 * rb) << 16;
    const float sc = LOG2E * 0.125f;
    const float2 sc2 = make_float2(sc, sc);
    const float NEG = -INFINITY;
    float m0 = NEG, m1 = NEG;
    // this thread's share of the row sums (its 16 columns of rows r0 and r1),
    // in the units of the running maxima m0, m1 (register row sums only)
    float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
    const float2 one2 = make_float2(1.f, 1.f);
    const int r0 = 16 * rb + g4, r1 = r0 + 8;  // query rows of this thread
    // stmatrix row address in P buffer 0: matrix mi = lane >> 3 of store jj
    // covers rows 16 rb + 8 (mi & 1) .. + 7 and 16-byte chunk 2 jj + (mi >> 1),
    // placed by the 128-byte swizzle at chunk ^ (row & 7); the buffer is
    // 1024-byte aligned, so store jj's address is p_addr ^ (jj << 5)
    uint32_t p_addr;
    {
      const uint32_t mi = (uint32_t)lane >> 3, rr = (uint32_t)lane & 7;
      const uint32_t R = (uint32_t)(16 * rb) + (mi & 1) * 8 + rr;
      p_addr = saddr(sm.p[0]) + R * 128u + (((mi >> 1) ^ rr) << 4);
    }
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
      const int s = i % BST, b = PTMEM ? (i & 1) : i % NSBUF, pb = PTMEM ? (i & 1) : i % PBUF;
      if (!mbar_wait_warp(&sm.s_full[b], (PTMEM ? (i >> 1) : i / NSBUF) & 1, abort_flag)) { ok = false; break; }
      fence_after();
      float sv[32];
      tmem_ld64(tmem + lane_off + s_addr(b), sv);
      if constexpr (!BIAS3) {
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[b]);
      }

      // scale, bias (log2 units) and row maxima; sv[4j], sv[4j+1] belong to
      // row r0 and sv[4j+2], sv[4j+3] to row r1
      float mx0, mx1;
      const bool nobias = sm.all_zero[s] != 0;
      if (nobias) {
        // complete kept tile: maxima of the raw scores (the scale is positive)
        mx0 = max_row<0>(sv) * sc;
        mx1 = max_row<2>(sv) * sc;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 bb = *reinterpret_cast<const float2*>(&sm.bias[s][8 * j + 2 * q4]);
          const float2 t0 = ffma2(make_float2(sv[4 * j + 0], sv[4 * j + 1]), sc2, bb);
          const float2 t1 = ffma2(make_float2(sv[4 * j + 2], sv[4 * j + 3]), sc2, bb);
          sv[4 * j + 0] = t0.x;
          sv[4 * j + 1] = t0.y;
          sv[4 * j + 2] = t1.x;
          sv[4 * j + 3] = t1.y;
        }
        mx0 = max_row<0>(sv);
        mx1 = max_row<2>(sv);
      }
      if constexpr (RING) {
        // this warp is done with the block's bias row
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.b_empty[s]);
      }
      if constexpr (BIAS3) {
        // done with the block's scores and its bias row
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[b]);
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      // lazy maximum: move it only when the block exceeds it by more than 8 (x256)
      const bool up0 = mx0 > m0 + 8.f, up1 = mx1 > m1 + 8.f;
      const float mn0 = up0 ? mx0 : m0, mn1 = up1 ? mx1 : m1;
      const float base0 = mn0 == NEG ? 0.f : mn0, base1 = mn1 == NEG ? 0.f : mn1;
      const float al0 = up0 ? fast_exp2(m0 - base0) : 1.f, al1 = up1 ? fast_exp2(m1 - base1) : 1.f;
      // p = 2^(scaled score - base): one packed FMA per two elements
      const float ka = nobias ? sc : 1.f;
      const float2 ka2 = make_float2(ka, ka);
      const float2 nb0 = make_float2(-base0, -base0), nb1 = make_float2(-base1, -base1);
      if (!RSUM_MMA) {
        ls0.x *= al0;
        ls0.y *= al0;
        ls1.x *= al1;
        ls1.y *= al1;
      }
      uint32_t pk[8][2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 e0 = ffma2(make_float2(sv[4 * j + 0], sv[4 * j + 1]), ka2, nb0);
        const float2 e1 = ffma2(make_float2(sv[4 * j + 2], sv[4 * j + 3]), ka2, nb1);
        float2 p0, p1;
        if (j >= 8 - EMU) {
          p0 = exp2_poly2(e0);
          p1 = exp2_poly2(e1);
        } else {
          p0 = make_float2(fast_exp2(e0.x), fast_exp2(e0.y));
          p1 = make_float2(fast_exp2(e1.x), fast_exp2(e1.y));
        }
        pk[j][0] = pack_bf16(p0.x, p0.y);
        pk[j][1] = pack_bf16(p1.x, p1.y);
        if (!RSUM_MMA) {
          // the row sums add exactly the bf16 values that O += P V multiplies
          ls0 = ffma2(make_float2(__uint_as_float(pk[j][0] << 16), __uint_as_float(pk[j][0] & 0xffff0000u)), one2,
                      ls0);
          ls1 = ffma2(make_float2(__uint_as_float(pk[j][1] << 16), __uint_as_float(pk[j][1] & 0xffff0000u)), one2,
                      ls1);
        }
      }
      m0 = mn0;
      m1 = mn1;
      if constexpr (PTMEM) {
        // P buffer b is free once PV of block i - 2 has read it
        if (i >= 2 && !mbar_wait_warp(&sm.pv_done[b], ((i >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        tmem_st_p(tmem + lane_off + p_addr_tmem(b), pk);
      } else {
        // P buffer pb is free once PV of block i-PBUF has completed
        if (i >= PBUF && !mbar_wait_warp(&sm.pv_done[pb], ((i / PBUF) - 1) & 1, abort_flag)) { ok = false; break; }
        const uint32_t poff = (uint32_t)pb * (64u * 64u * 2u);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          stmatrix4((p_addr ^ ((uint32_t)jj << 5)) + poff, pk[2 * jj][0], pk[2 * jj][1], pk[2 * jj + 1][0],
                    pk[2 * jj + 1][1]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // rescale O and L (TMEM) when any row of this warp moved its maximum
      if (i >= 1 && __any_sync(0xffffffffu, up0 || up1)) {
        const int jp = i - 1;
        if (!mbar_wait_warp(&sm.pv_done[PTMEM ? (jp & 1) : jp % PBUF], (PTMEM ? (jp >> 1) : jp / PBUF) & 1,
                            abort_flag)) { ok = false; break; }
        fence_after();
        float o[32];
        tmem_ld64(tmem + lane_off + COL_O, o);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          o[4 * j + 0] *= al0;
          o[4 * j + 1] *= al0;
          o[4 * j + 2] *= al1;
          o[4 * j + 3] *= al1;
        }
        tmem_st64(tmem + lane_off + COL_O, o);
        if (RSUM_MMA) {
          float lv[4];
          tmem_ld8(tmem + lane_off + LANE_L + COL_O, lv);
          lv[0] *= al0;
          lv[1] *= al0;
          lv[2] *= al1;
          lv[3] *= al1;
          tmem_st8(tmem + lane_off + LANE_L + COL_O, lv);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[pb]);
    }
    // ---------------- epilogue ----------------
    if (ok && nb >= 1 &&
        !mbar_wait_warp(&sm.pv_done[PTMEM ? ((nb - 1) & 1) : (nb - 1) % PBUF],
                        (PTMEM ? ((nb - 1) >> 1) : (nb - 1) / PBUF) & 1, abort_flag))
      ok = false;
    if (ok) {
      fence_after();
      float o[32];
      float l0 = 0.f, l1 = 0.f;   // row sums (every column of L holds the row's sum)
      if (nb >= 1) {
        tmem_ld64(tmem + lane_off + COL_O, o);
        if (RSUM_MMA) {
          float lv[4];
          tmem_ld8(tmem + lane_off + LANE_L + COL_O, lv);
          l0 = lv[0];
          l1 = lv[2];
        } else {
          // the four threads of a quad hold the 64 columns of rows r0 and r1
          l0 = ls0.x + ls0.y;
          l1 = ls1.x + ls1.y;
          l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
          l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
          l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
          l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.f;
      }
      if constexpr (MODE == 1) {
        // split partials: unnormalised output, row maximum (log2 units) and row sum
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = half ? r1 : r0;
          const size_t row = ((size_t)sp * g.H + h) * g.NSp + (size_t)qb * 64 + r;
          float* po = a.part_o + row * D;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float2*>(po + 8 * j + 2 * q4) = make_float2(o[4 * j + half * 2], o[4 * j + half * 2 + 1]);
          if (q4 == 0) *reinterpret_cast<float2*>(a.part_ml + row * 2) = make_float2(half ? m1 : m0, half ? l1 : l0);
        }
      } else if (!own_kept) {
        // exact self key + landmark of the other n_t - 1 tokens of the own tile
        const size_t tb = ((size_t)h * g.T + t) * TOK * D;                                 // Q: 64-row tiles
        const size_t kb = PACK ? (size_t)sm.own_kv_row * D : tb;                           // K, V
        const __nv_bfloat16* Qp = static_cast<const __nv_bfloat16*>(a.Qp) + tb;
        const __nv_bfloat16* Kp = static_cast<const __nv_bfloat16*>(a.Kp) + kb;
        const __nv_bfloat16* Vp = static_cast<const __nv_bfloat16*>(a.Vp) + kb;
        const float* km = a.km + ((size_t)h * g.T + t) * D;
        const float* vm = a.vm + ((size_t)h * g.T + t) * D;
        const float nt = (float)n_t;
        const float inv = n_t > 1 ? 1.0f / (float)(n_t - 1) : 0.f;
        const float lnb = n_t > 1 ? a.ln_tab[n_t - 1] * LOG2E : 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = half ? r1 : r0;
          float qk = 0.f, qm = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 8 * j + 2 * q4 + e;
              const float qv = __bfloat162float(Qp[r * D + c]);
              qk = fmaf(qv, __bfloat162float(Kp[r * D + c]), qk);
              qm = fmaf(qv, km[c], qm);
            }
          }
          qk += __shfl_xor_sync(0xffffffffu, qk, 1);
          qk += __shfl_xor_sync(0xffffffffu, qk, 2);
          qm += __shfl_xor_sync(0xffffffffu, qm, 1);
          qm += __shfl_xor_sync(0xffffffffu, qm, 2);
          const float s_self = qk * sc;
          const float s_lm = n_t > 1 ? (nt * qm - qk) * inv * sc + lnb : NEG;
          float& m = half ? m1 : m0;
          float& l = half ? l1 : l0;
          const float mn = fmaxf(m, fmaxf(s_self, s_lm));
          const float al = fast_exp2(m - mn), ps = fast_exp2(s_self - mn);
          const float pl = n_t > 1 ? fast_exp2(s_lm - mn) : 0.f;
          m = mn;
          l = l * al + ps + pl;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 8 * j + 2 * q4 + e;
              const float vv = __bfloat162float(Vp[r * D + c]);
              const float vl = (nt * vm[c] - vv) * inv;
              float& oo = o[4 * j + half * 2 + e];
              oo = oo * al + ps * vv + pl * vl;
            }
          }
        }
      }
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
#pragma unroll
      for (int half = 0; half < 2 && MODE == 0; ++half) {
        const int r = half ? r1 : r0;
        if (r >= n_t) continue;
        const float il = 1.0f / (half ? l1 : l0);
        __nv_bfloat16* dst = out + (tile_token(g, ts, r) * g.H + h) * D;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = 8 * j + 2 * q4;
          *reinterpret_cast<__nv_bfloat162*>(dst + c) =
              __floats2bfloat162_rn(o[4 * j + half * 2] * il, o[4 * j + half * 2 + 1] * il);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

}  // namespace tc

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 map over [rows, 64] with a 64 x box_rows box and 128-byte swizzle
static bool make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned box_rows = 64) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rows == 0) rows = 64;  // never read: keep the encoder happy
  cuuint64_t dims[2] = {64, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Launches the tcgen05 kernel for every work item of `mode` (0: patch rows of
// the sparse stage, one per (head, query tile); 1: special-token rows, one per
// (head, key split, query block)).
static int launch_tc(const AttnArgs& a, int mode, cudaStream_t st) {
  const Geo& g = a.g;
  const long long items = mode == 0 ? (long long)g.T * g.H : (long long)(g.NSp / 64) * g.H * a.splits;
  if (items == 0 || g.T == 0) return ZEBRA_OK;
  tc::Params p;
  p.a = a;
  const unsigned long long tile_rows = (unsigned long long)g.H * g.T * 64;
  const unsigned long long spec_rows = (unsigned long long)g.H * g.NSp;
  const unsigned long long dense_rows = (unsigned long long)g.H * g.V * g.RPV;   // K, V: dense layout, 8-row groups
  bool ok = make_map(&p.tq, a.Qp, tile_rows) &&
            make_map(&p.tkl, a.Kl, (unsigned long long)g.H * g.Tpad) &&
            make_map(&p.tvl, a.Vl, (unsigned long long)g.H * g.Tpad) && make_map(&p.tks, a.Ks, spec_rows) &&
            make_map(&p.tvs, a.Vs, spec_rows) && make_map(&p.tqs, a.Qs, spec_rows);
  for (unsigned m = 0; m < 8 && ok; ++m)
    ok = make_map(&p.tkg[m], a.Kp, dense_rows, 8 * (m + 1)) && make_map(&p.tvg[m], a.Vp, dense_rows, 8 * (m + 1));
  if (!ok) {
    set_error("cuTensorMapEncodeTiled failed");
    return ZEBRA_ERR_CUDA;
  }
  const bool pack = (g.Hp % TILE) != 0 || (g.Wp % TILE) != 0;   // partial tiles to pack
  auto kern = mode == 0 ? (pack ? tc::attn_tc_kernel<0, true> : tc::attn_tc_kernel<0, false>)
                        : (pack ? tc::attn_tc_kernel<1, true> : tc::attn_tc_kernel<1, false>);
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::SMEM_BYTES);
  // Work items go out in launches of one resident wave each. All CTAs of a
  // launch start together and walk their key blocks in ascending order at
  // about the same rate, so at any moment they read K/V tiles from a narrow
  // window of tile indices that stays in L2. In one launch of all items the
  // CTAs of later waves start whenever a slot frees up, their positions spread
  // over the whole key range, and most K/V reads go to DRAM (sparse rows at
  // 1,024 views x 16 heads: 25% slower, the extra DRAM power pulling the clock
  // down under the board's power limit).
  long long wave = items;
  {
    // the kernel is built for CTAS_PER_SM resident CTAs per SM (registers,
    // shared memory and TMEM columns are sized for it)
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        sms > 0)
      wave = (long long)tc::CTAS_PER_SM * sms;
    cudaGetLastError();
  }
  ProfScope prof(mode == 0 ? "attn_sparse_rows" : "attn_special_rows", st);
  prof.set_launches((int)((items + wave - 1) / wave));
  for (long long base = 0; base < items; base += wave) {
    p.item0 = (int)base;
    const unsigned n = (unsigned)(items - base < wave ? items - base : wave);
    kern<<<n, tc::THREADS, tc::SMEM_BYTES, st>>>(p);
    count_launch();
    if (int rc = check_launch(mode == 0 ? "attn_tc_kernel<patch rows>" : "attn_tc_kernel<special rows>")) return rc;
  }
  return ZEBRA_OK;
}

int launch_sparse_attn_tc(const AttnArgs& a, cudaStream_t st) { return launch_tc(a, 0, st); }
int launch_special_rows_tc(const AttnArgs& a, cudaStream_t st) { return launch_tc(a, 1, st); }

}  // namespace zebra
