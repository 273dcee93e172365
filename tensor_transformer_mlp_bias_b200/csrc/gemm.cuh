// Persistent, warp-specialised tcgen05 GEMM with the MLP block's fused
// epilogues, for sm_100a.
//
//   D[M,N] = sum_k Aop[M,k] · Bop[k,N]   (bf16 in, fp32 accumulate in TMEM)
//
// Persistent grid, one CTA per SM.  In the default pair mode two CTAs of a
// cluster share each 256x256 output tile through the 2-SM tensor-core
// instruction (cta_group::2): CTA r of the pair owns rows [128r, 128r+128)
// of the tile (its half of the A operand and of the TMEM accumulator) and
// columns [128r, 128r+128) of the B operand, so each SM streams half of B
// instead of all of it.  In single mode a CTA owns a 128x256 tile alone.
// Warp roles (per CTA):
//   warp 0      TMA producer: fills a ring of STAGES shared-memory stages
//               (its A rows x 64 and its B rows x 64, 128-byte swizzle); the
//               pair leader arms the "full" mbarrier with the byte count of
//               both CTAs' loads, which all complete on the leader's barrier;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators
//               per CTA); on the leader, one thread issues tcgen05.mma
//               (M=256 across the pair, or 128 alone; N=256; K=16) per
//               16-wide K slice, committing each stage back to the "empty"
//               barriers of both CTAs and each finished accumulator to their
//               "tmem full" barriers;
//   warps 2-    epilogue (8 or 16 warps, see TileCfg):
//               tcgen05.ld the accumulator (one row per thread, 32 columns
//               per load), apply the fused math, store to global memory,
//               release the accumulator.
// The two accumulators let the epilogue of one unit overlap the mainloop of
// the next.
//
// Shard reduction (EPI_SHARD_SUM).  For the row-parallel GEMM and for the
// input gradient of the column-parallel GEMM, K is the concatenation of t
// shard segments.  Each segment is accumulated into a fresh TMEM accumulator
// (the accumulate flag restarts at the segment's first K slice), so the
// epilogue receives the t shard partials P_0..P_{t-1} separately and sums
// them in registers in ascending shard order, adds the bias and rounds once.
// This is the on-device stand-in for the tensor-parallel all-reduce.
//
// Split operands.  An activation or gradient that is computed here (H, dH)
// is kept as a bf16 pair v = hi + lo (hi = bf16(v), lo = bf16(v - hi), about
// 16 significant bits).  A product that must see that precision runs its K
// loop twice ("parts"): once over (hi, other operand) and once over
// (lo, other operand), accumulating into the same TMEM accumulator.  With
// DUAL, the split operand is A and both halves ride in the same stage: one
// pass over K loads A_hi, A_lo and B once and issues both products per K
// slice, so B crosses from L2 once instead of twice.
//
// Operand layouts.  A K-major operand is stored [rows, K] with K contiguous
// and arrives as one TMA box of 64 (K) x rows.  An MN-major operand is
// stored [K, rows] with rows contiguous and arrives as 64-row-wide boxes of
// 64 (rows) x 64 (K); the MMA reads it through an MN-major descriptor, so no
// transpose is ever materialised.
//
// 8-bit residual products (F8LO).  In the fp16 + e4m3 mode (fp8.cuh) a
// weight gradient is one fp16 product plus an e4m3 residual product into the
// same accumulator.  The K loop runs the fp16 part (64-token stages) and then
// the e4m3 part in stages of 128 tokens, which take the same bytes: A and B
// arrive as 128 (rows) x 128 (K) boxes, 128-byte rows, and each stage issues
// four kind::f8f6f4 MMAs of K = 32 per MMA width.
//
// Cross-GPU shard reduction (EPI_PEER).  With the block sharded over several
// GPUs, a rank's row-parallel GEMM sends each 128-row block of its fp32
// partial straight to the GPU that owns those token rows (peer.cuh): plain
// coalesced stores over NVLink from the epilogue, then a per-tile arrival
// count raised at system scope; the owner's reduce kernel sums the partials.
//
// Every wait is bounded (see mbar_wait).  A wait that runs out records
// status 7 (timeout) in the device status word, raises a CTA-wide abort
// flag so the other roles leave their loops, and the CTA still drains its
// in-flight TMA copies and tensor-core operations and frees its TMEM before
// returning.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "fp8.cuh"
#include "peer.cuh"
#include "ptx.cuh"

namespace mlptp {

constexpr int BM = 128;  // accumulator rows per CTA
constexpr int BN = 256;  // accumulator columns
constexpr int BK = 64;
constexpr int MN_BOX_BYTES = 64 * BK * 2;   // one 64x64 bf16 box, 8 KB
constexpr int F8_BOX_BYTES = 128 * 2 * BK;  // one 128x128 e4m3 box, 16 KB
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int CTL_BYTES = 1024;

enum Epi : int { EPI_BIAS_GELU = 0, EPI_SHARD_SUM = 1, EPI_GELU_GRAD = 2, EPI_STORE = 3, EPI_PEER = 4 };

// Epilogue staging per epilogue warp: one 32x32 tile per output, laid out
// for the TMA store (bf16: 64-byte rows, 64-byte swizzle; fp32: 128-byte
// rows, 128-byte swizzle).
constexpr int EPI_BF16_TILE = 32 * 32 * 2;
constexpr int EPI_F32_TILE = 32 * 32 * 4;
__host__ __device__ constexpr int epi_warp_bytes(int epi) {
  return epi == EPI_BIAS_GELU ? EPI_F32_TILE + 2 * EPI_BF16_TILE
                              : (epi == EPI_GELU_GRAD ? 2 * EPI_BF16_TILE
                                                      : (epi == EPI_PEER ? EPI_F32_TILE : EPI_BF16_TILE));
}

// Tile shape.  TN is the number of output columns per tile: 256 (one MMA
// width, two TMEM accumulators so the epilogue overlaps the next tile) or
// 512 (pair mode only: two MMA widths side by side, one accumulator filling
// all 512 TMEM columns).  The wide tile reads 25% fewer operand bytes per
// FLOP from L2, which is what bounds these GEMMs without TMA multicast.
// STAGES is the shared-memory pipeline depth (BK-wide K slices in flight):
// as many as fit beside the epilogue staging.  EW is the number of epilogue
// warps, 8 or 16: four lane quadrants times 2 or 4 column slices.  Sixteen
// keep twice as many chunks in flight per scheduler, which pays where the
// epilogue (waiting on TMEM and global loads) outlasts a short mainloop, at
// the cost of staging space, i.e. pipeline stages.
template <bool PAIR, int TN, int EPI, int EW = 8, bool DUAL = false>
struct TileCfg {
  static_assert(TN == 256 || (TN == 512 && PAIR), "wide tiles need a CTA pair");
  static constexpr int CTAS = PAIR ? 2 : 1;
  static constexpr int TILE_M = BM * CTAS;                    // output rows per tile
  static constexpr int TILE_N = TN;
  static constexpr int WIDTHS = TN / BN;                       // MMA widths per tile
  static constexpr int ACCS = TN == 256 ? 2 : 1;               // TMEM accumulators (double-buffered or not)
  static constexpr int SUB_ROWS = PAIR ? BN / 2 : BN;          // B rows per CTA per MMA width
  static constexpr int B_ROWS = SUB_ROWS * WIDTHS;             // B operand rows held by one CTA
  static constexpr int SUB_BYTES = SUB_ROWS * BK * 2;
  static constexpr int B_STAGE_BYTES = B_ROWS * BK * 2;
  static constexpr int A_BYTES = A_STAGE_BYTES * (DUAL ? 2 : 1);      // A (and A_lo with DUAL)
  static constexpr int STAGE_BYTES = A_BYTES + B_STAGE_BYTES;          // one CTA's share of a stage
  static constexpr int EPI_WARPS = EW;
  static constexpr int THREADS = 64 + EPI_WARPS * 32;          // producer, MMA issuer, epilogue
  static constexpr int SLICE_COLS = TN / (EPI_WARPS / 4);      // columns per epilogue warp (4 lane quadrants)
  static_assert(EPI_WARPS % 4 == 0 && SLICE_COLS % 32 == 0, "epilogue warps must tile the accumulator");
  static constexpr int EPI_BYTES = EPI_WARPS * epi_warp_bytes(EPI);
  static constexpr int SMEM_LIMIT = 227 * 1024;
  static constexpr int FIXED = EPI_BYTES + CTL_BYTES + 1024;   // + alignment slack
  static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(STAGES >= 3, "pipeline too shallow");
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED;
};

constexpr unsigned int STATUS_TIMEOUT = 7u;
constexpr unsigned int STATUS_BOUNDS = 8u;

// Bounds-checking build (compiled with -DMLPTP_BOUNDS_CHECK): every plain
// global access that does not go through a tensor map checks the last
// element it touches against its buffer's element count.  A bad index
// records status 8 and the access site in the status word and skips the
// access (no trap, no device assert).  In the normal build the check
// compiles away.
__device__ __forceinline__ bool index_ok(long long last, long long n, unsigned int* status, unsigned int site) {
#ifdef MLPTP_BOUNDS_CHECK
  if (last < 0 || last >= n) {
    atomicCAS(status, 0u, STATUS_BOUNDS);
    atomicCAS(status + 1, 0u, site);
    return false;
  }
#else
  (void)last;
  (void)n;
  (void)status;
  (void)site;
#endif
  return true;
}

struct GemmParams {
  int M, N;
  int shards;             // K segments reduced in the epilogue (EPI_SHARD_SUM); 1 otherwise
  // Work list.  Without a K split: tiles [0, full_tiles) whole; each later
  // tile (the partial last wave of a shard-sum GEMM) as tail_split pieces of
  // shards/tail_split consecutive shards.  With a K split (kb_split > 1, GEMMs
  // without shards and with fewer tiles than CTA pairs): every tile as
  // kb_split pieces of consecutive K slices.  A piece's fp32 sum goes to
  // tail_scratch and a separate kernel adds the pieces of a tile in order.
  int full_tiles, tail_split, kb_split, num_work;
  float* tail_scratch;    // [pieces][TILE_M][TILE_N] fp32
  long long scratch_elems;  // floats in tail_scratch (bounds-checking build)
  int parts;              // 1, or 2 when an operand is a bf16 (hi, lo) pair
  int kblocks_per_shard;  // BK-wide K slices per segment and part (F8LO: of the fp16 part)
  int kb_per_unit;        // K slices (stages) per segment over all parts
  int m_blocks, n_blocks, num_tiles, group_m;
  __nv_bfloat16* out0;        // H_hi | Y | dH_hi | dX | dA | dB
  __nv_bfloat16* out1;        // H_lo (EPI_BIAS_GELU) | dH_lo (EPI_GELU_GRAD)
  float* out_f32;             // Z (EPI_BIAS_GELU)
  float* colsum;              // [row blocks*4, N] column sums of dH (EPI_GELU_GRAD), may be null
  long long colsum_elems;     // floats in colsum (bounds-checking build)
  const __nv_bfloat16* bias;  // a (EPI_BIAS_GELU) or b (EPI_SHARD_SUM), may be null for the latter
  const float* aux;           // Z (EPI_GELU_GRAD)
  unsigned int* status;       // device status word pair in the workspace
  unsigned long long budget_ns;
  unsigned int debug_flags;
  PeerParams peer;            // EPI_PEER: where each row block's partial goes
  long long peer_recv_elems;  // floats in each receive buffer (bounds-checking build)
  // fp16 + e4m3 mode (fp8.cuh)
  uint32_t f16_ops;                // kind::f16 operands are fp16 (1) or bf16 (0)
  const unsigned int* fp8_stats;   // the mode's statistics, from which the scales follow (NULL: none)
  int out_scale;                   // OUT_SCALE_*: factor on the accumulator before the output rounding
  int fp8_out;                     // EPI_BIAS_GELU / EPI_GELU_GRAD: out0 fp16, out1 e4m3 residual
};

enum OutScale : int { OUT_SCALE_NONE = 0, OUT_SCALE_INV_SY = 1, OUT_SCALE_INV_SX_SH = 2, OUT_SCALE_INV_SH = 3 };

// The output factor that undoes the operands' power-of-two scales.
__device__ __forceinline__ float out_factor(const GemmParams& p) {
  if (p.fp8_stats == nullptr || p.out_scale == OUT_SCALE_NONE) return 1.0f;
  const Fp8Scales sc = fp8_scales(p.fp8_stats);
  if (p.out_scale == OUT_SCALE_INV_SY) return 1.0f / sc.sY;
  if (p.out_scale == OUT_SCALE_INV_SX_SH) return 1.0f / (sc.sX * sc.sH);
  return 1.0f / sc.sH;
}

__device__ __forceinline__ void record_range(const GemmParams& p, bool bad, unsigned int site) {
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) {
    atomicCAS(p.status, 0u, STATUS_RANGE);
    atomicCAS(p.status + 1, 0u, site);
  }
}

// Tensor maps of the operands, one per K part (part 1 repeats part 0 for an
// operand that is not split), and of the outputs (32x32 store boxes):
// out[0] = out0, out[1] = out1 (bf16), out[2] = out_f32.
struct GemmMaps {
  CUtensorMap a[2];
  CUtensorMap b[2];
  CUtensorMap out[3];
};

constexpr int MAX_STAGES = 8;
struct GemmCtl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(GemmCtl) <= CTL_BYTES, "control block too large");

// Tile order: groups of `group_m` row blocks; inside a group the row block
// varies fastest.  group_m = m_blocks walks all row blocks of one column
// block before the next (the row operand stays in L2); group_m = 1 walks
// columns fastest.
__device__ __forceinline__ void tile_coords(int tile, const GemmParams& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.n_blocks;
  const int g = tile / per_group;
  const int first_m = g * p.group_m;
  const int gsz = min(p.m_blocks - first_m, p.group_m);
  const int r = tile - g * per_group;
  mb = first_m + r % gsz;
  nb = r / gsz;
}

// One item of the work list: a whole tile (piece < 0) or one piece of a
// split tile: shards [s_begin, s_end) and, within each shard, the K slices
// [i_begin, i_end) of the parts x K-blocks loop.
struct WorkItem {
  int tile, s_begin, s_end, i_begin, i_end, piece;
};

__device__ __forceinline__ WorkItem work_item(int w, const GemmParams& p, int kb_per_unit) {
  if (p.kb_split > 1) {
    const int chunk = w % p.kb_split;
    return WorkItem{w / p.kb_split, 0, p.shards, chunk * kb_per_unit / p.kb_split,
                    (chunk + 1) * kb_per_unit / p.kb_split, w};
  }
  if (w < p.full_tiles) return WorkItem{w, 0, p.shards, 0, kb_per_unit, -1};
  const int piece = w - p.full_tiles;
  const int per = p.shards / p.tail_split;
  const int part = piece % p.tail_split;
  return WorkItem{p.full_tiles + piece / p.tail_split, part * per, part * per + per, 0, kb_per_unit, piece};
}

__device__ __forceinline__ void record_timeout(const GemmParams& p, volatile int* abort, unsigned int where) {
  *abort = 1;
  atomicCAS(p.status, 0u, STATUS_TIMEOUT);
  atomicCAS(p.status + 1, 0u, where);
}

// Bounded wait that ignores the abort flag (used only to drain the CTA's own
// in-flight asynchronous work before it exits).
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, uint64_t budget_ns) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 0;; ++n) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((n & 31u) == 31u && global_timer_ns() - t0 > budget_ns) return false;
  }
}

// ---------------------------------------------------------------- math
// tanh-form GeLU written through the logistic function:
//   ½(1 + tanh u) = σ(2u),  u = √(2/π)(x + 0.044715 x³)
//   g(x)  = x·σ(2u)
//   g'(x) = σ(2u)·(1 + 2x(1 − σ(2u))·√(2/π)(1 + 3·0.044715 x²))
// (1 − tanh²u = 4σ(1 − σ)); this form has no cancellation for x << 0.
__device__ __forceinline__ float sigmoid2u(float x, float& du) {
  const float c = 0.7978845608028654f;
  const float k = 0.044715f;
  const float x2 = x * x;
  const float u = c * fmaf(k * x2, x, x);
  du = c * fmaf(3.0f * k, x2, 1.0f);
  return __fdividef(1.0f, 1.0f + __expf(-2.0f * u));
}

__device__ __forceinline__ float gelu_f(float x) {
  float du;
  return x * sigmoid2u(x, du);
}

__device__ __forceinline__ float gelu_grad_f(float x) {
  float du;
  const float s = sigmoid2u(x, du);
  return s * fmaf(2.0f * x * (1.0f - s), du, 1.0f);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t v) {
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v);
  return __bfloat1622float2(b);
}

// v0, v1 -> (hi pair, lo pair): hi = bf16(v), lo = bf16(v - hi).
__device__ __forceinline__ void split_bf16x2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(v0, v1);
  const float2 h = unpack_bf16x2(hi);
  lo = pack_bf16x2(v0 - h.x, v1 - h.y);
}

// 32 consecutive bf16 values: raw 16-byte loads, then widening to fp32.
__device__ __forceinline__ void load_bf16x32_raw(const __nv_bfloat16* src, uint4 (&w)[4]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < 4; ++v) w[v] = __ldg(s + v);
}

__device__ __forceinline__ void widen_bf16x32(const uint4 (&w)[4], float (&dst)[32]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t u[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(u[e]);
      dst[v * 8 + 2 * e] = f.x;
      dst[v * 8 + 2 * e + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&dst)[32]) {
  uint4 w[4];
  load_bf16x32_raw(src, w);
  widen_bf16x32(w, dst);
}

// Row `r` (this lane) of a 32x32 bf16 staging tile: 64-byte rows, 16-byte
// chunk j stored at chunk j ^ ((r >> 1) & 3) (the TMA 64-byte swizzle; the
// tile is 512-byte aligned), so a warp's 16-byte stores hit every bank.
__device__ __forceinline__ void stage_bf16x32(uint32_t tile, int r, const uint32_t (&packed)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_shared_v4(tile + r * 64 + ((j ^ ((r >> 1) & 3)) << 4), packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                 packed[4 * j + 3]);
}

// Row `r` of a 32x32 fp32 staging tile: 128-byte rows, chunk j stored at
// chunk j ^ (r & 7) (the TMA 128-byte swizzle; the tile is 1024-byte aligned).
__device__ __forceinline__ void stage_f32x32(uint32_t tile, int r, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(tile + r * 128 + ((j ^ (r & 7)) << 4), __float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                 __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
}

// This lane's row of the 32x32 fp32 block at (row0, col) of a row-major
// [M, N] matrix, read coalesced: eight lanes cover one 128-byte row segment
// (4 rows per load instruction, 8 instructions), the block is transposed
// through `tile` (4 KB of the warp's staging, free on entry: 128-byte rows,
// chunk j of row r at chunk j ^ (r & 7), so both the writes and the per-row
// reads hit every bank), and each lane reads back its own row.  Reading the
// rows one per lane instead touches 32 cache lines per instruction.  Rows
// at or past M read as 0.  `tile` is free again on return.
__device__ __forceinline__ void load_rows_f32x32_coalesced(const float* src, int M, int N, int row0, int col,
                                                           uint32_t tile, int lane, float (&dst)[32]) {
  const int rr = lane >> 3, cc = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = i * 4 + rr;
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (row0 + r < M)
      v = __ldg(reinterpret_cast<const float4*>(src + static_cast<size_t>(row0 + r) * static_cast<size_t>(N) + col) + cc);
    st_shared_v4(tile + r * 128 + ((cc ^ (r & 7)) << 4), __float_as_uint(v.x), __float_as_uint(v.y),
                 __float_as_uint(v.z), __float_as_uint(v.w));
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 v = ld_shared_v4f(tile + lane * 128 + ((j ^ (lane & 7)) << 4));
    dst[4 * j] = v.x;
    dst[4 * j + 1] = v.y;
    dst[4 * j + 2] = v.z;
    dst[4 * j + 3] = v.w;
  }
  __syncwarp();
}

// Column sums over the warp's 32 rows: lane r holds row r's 32 values; on
// return lane j holds the sum over rows of column j.  Recursive halving:
// at each step a lane keeps the half of its columns selected by one bit of
// its lane index and adds the partner lane's copy of that half (31 shuffles
// in all, fixed order, so the result is deterministic).
__device__ __forceinline__ float warp_column_sums(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step;           // values kept after this step
    const bool upper = (lane & half) != 0;  // keep the upper half of the current columns
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = upper ? v[j] : v[j + half];
      const float keep = upper ? v[j + half] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

// ---------------------------------------------------------------- kernel
template <bool A_MN, bool B_MN, int EPI, bool PAIR, int TN, int EW, bool DUAL, bool F8LO>
__global__ void __launch_bounds__(TileCfg<PAIR, TN, EPI, EW, DUAL>::THREADS, 1)
    mlp_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using Cfg = TileCfg<PAIR, TN, EPI, EW, DUAL>;
  static_assert(!DUAL || PAIR, "both halves of A in one stage: pair mode");
  static_assert(!F8LO || (A_MN && B_MN && !DUAL && EPI == EPI_STORE),
                "8-bit residual products: weight gradients over MN-major operands");
  static_assert(EPI != EPI_SHARD_SUM || TN == 256, "the shard sum is held in registers for 256 columns");
  static_assert(EPI != EPI_PEER || (TN == 256 && EW == PEER_ARRIVALS),
                "a peer tile block is one MMA width and its arrival count is one per epilogue warp");
  constexpr int ACCS = Cfg::ACCS;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sEpi = smem + STAGES * Cfg::STAGE_BYTES;  // 1024-aligned: STAGE_BYTES is a multiple of 1024
  GemmCtl* ctl = reinterpret_cast<GemmCtl*>(sEpi + Cfg::EPI_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_cta_rank() : 0u;  // position in the CTA pair
  const bool leader = rank == 0;
  const int cluster_id = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int num_clusters = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);   // one arrival: the leader's expect_tx
      mbar_init(&ctl->empty[s], 1);  // one arrival: the leader's MMA commit
    }
#pragma unroll
    for (int a = 0; a < ACCS; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], Cfg::EPI_WARPS * Cfg::CTAS);  // every epilogue warp of the pair
    }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      prefetch_tensormap(&maps.a[i]);
      prefetch_tensormap(&maps.b[i]);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  if constexpr (PAIR) {
    cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  // Everything above touches only this CTA's shared memory, TMEM and the
  // kernel parameters, so it may overlap the previous kernel's tail; every
  // global read and write below comes after the previous grid completed.
  grid_launch_dependents();
  grid_wait_prerequisites();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const uint64_t budget = p.budget_ns;
  const int kb_per_unit = p.kb_per_unit;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: armed at least once / parity of last arming
      bool ok = true;
      bool first = true;
      for (int w = cluster_id; ok && w < p.num_work; w += num_clusters) {
        const WorkItem it = work_item(w, p, kb_per_unit);
        int mb, nb;
        tile_coords(it.tile, p, mb, nb);
        const int m0 = mb * Cfg::TILE_M + static_cast<int>(rank) * BM;  // this CTA's A rows
        // this CTA's B rows for MMA width w start at n0 + w * BN
        const int n0 = nb * Cfg::TILE_N + static_cast<int>(rank) * Cfg::SUB_ROWS;
        for (int s = it.s_begin; ok && s < it.s_end; ++s) {
          for (int i = it.i_begin; i < it.i_end; ++i) {
            if ((p.debug_flags & 1u) && !first) {
              ok = false;  // test hook: stop feeding the tensor core after one stage
              break;
            }
            first = false;
            if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, budget)) {
              record_timeout(p, abort_flag, 0x100u);
              ok = false;
              break;
            }
            const bool f8 = F8LO && i >= p.kblocks_per_shard;  // an e4m3 stage of 2*BK tokens
            const int part = F8LO ? (f8 ? 1 : 0) : i / p.kblocks_per_shard;
            const int k0 = F8LO ? (f8 ? (i - p.kblocks_per_shard) * 2 * BK : i * BK)
                                : (s * p.kblocks_per_shard + (i - part * p.kblocks_per_shard)) * BK;
            const CUtensorMap* ma = &maps.a[part];
            const CUtensorMap* mbp = &maps.b[part];
            const uint32_t a_dst = smem_u32(sA + stage * Cfg::A_BYTES);
            const uint32_t b_dst = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
            if (f8) {
              // same bytes as a 16-bit stage: A 128 x 128, B per MMA width SUB_ROWS x 128
              uint32_t fb;
              if constexpr (PAIR) {
                fb = map_shared_to_cta(smem_u32(&ctl->full[stage]), 0u);
                if (leader) mbar_arrive_expect_tx(&ctl->full[stage], Cfg::CTAS * Cfg::STAGE_BYTES);
              } else {
                fb = smem_u32(&ctl->full[stage]);
                mbar_arrive_expect_tx(&ctl->full[stage], Cfg::STAGE_BYTES);
              }
              if (leader || !PAIR) {
                issued_mask |= 1u << stage;
                issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
              }
              if constexpr (PAIR) {
                tma_load_2d_pair(a_dst, ma, fb, m0, k0);
              } else {
                tma_load_2d(a_dst, ma, fb, m0, k0);
              }
#pragma unroll
              for (int w = 0; w < Cfg::WIDTHS; ++w)
#pragma unroll
                for (int j = 0; j < Cfg::SUB_ROWS / 128; ++j) {
                  if constexpr (PAIR) {
                    tma_load_2d_pair(b_dst + w * Cfg::SUB_BYTES + j * F8_BOX_BYTES, mbp, fb, n0 + w * BN + 128 * j, k0);
                  } else {
                    tma_load_2d(b_dst + w * Cfg::SUB_BYTES + j * F8_BOX_BYTES, mbp, fb, n0 + w * BN + 128 * j, k0);
                  }
                }
            } else if constexpr (PAIR) {
              const uint32_t fb = map_shared_to_cta(smem_u32(&ctl->full[stage]), 0u);
              if (leader) {
                mbar_arrive_expect_tx(&ctl->full[stage], Cfg::CTAS * Cfg::STAGE_BYTES);
                issued_mask |= 1u << stage;
                issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
              }
              if (A_MN) {
                tma_load_2d_pair(a_dst, ma, fb, m0, k0);
                tma_load_2d_pair(a_dst + MN_BOX_BYTES, ma, fb, m0 + 64, k0);
                if constexpr (DUAL) {  // the low half of A, same rows and K slice
                  tma_load_2d_pair(a_dst + A_STAGE_BYTES, &maps.a[1], fb, m0, k0);
                  tma_load_2d_pair(a_dst + A_STAGE_BYTES + MN_BOX_BYTES, &maps.a[1], fb, m0 + 64, k0);
                }
              } else {
                tma_load_2d_pair(a_dst, ma, fb, k0, m0);
                if constexpr (DUAL) tma_load_2d_pair(a_dst + A_STAGE_BYTES, &maps.a[1], fb, k0, m0);
              }
#pragma unroll
              for (int w = 0; w < Cfg::WIDTHS; ++w) {
                if (B_MN) {
#pragma unroll
                  for (int j = 0; j < Cfg::SUB_ROWS / 64; ++j)
                    tma_load_2d_pair(b_dst + w * Cfg::SUB_BYTES + j * MN_BOX_BYTES, mbp, fb, n0 + w * BN + 64 * j, k0);
                } else {
                  tma_load_2d_pair(b_dst + w * Cfg::SUB_BYTES, mbp, fb, k0, n0 + w * BN);
                }
              }
            } else {
              const uint32_t fb = smem_u32(&ctl->full[stage]);
              mbar_arrive_expect_tx(&ctl->full[stage], Cfg::STAGE_BYTES);
              issued_mask |= 1u << stage;
              issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
              if (A_MN) {
                tma_load_2d(a_dst, ma, fb, m0, k0);
                tma_load_2d(a_dst + MN_BOX_BYTES, ma, fb, m0 + 64, k0);
              } else {
                tma_load_2d(a_dst, ma, fb, k0, m0);
              }
#pragma unroll
              for (int w = 0; w < Cfg::WIDTHS; ++w) {
                if (B_MN) {
#pragma unroll
                  for (int j = 0; j < Cfg::SUB_ROWS / 64; ++j)
                    tma_load_2d(b_dst + w * Cfg::SUB_BYTES + j * MN_BOX_BYTES, mbp, fb, n0 + w * BN + 64 * j, k0);
                } else {
                  tma_load_2d(b_dst + w * Cfg::SUB_BYTES, mbp, fb, k0, n0 + w * BN);
                }
              }
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // No TMA write may still be landing in shared memory when the CTAs
      // exit: the barrier owner waits for the last arming of every stage
      // (immediate when the tensor-core warp already consumed it).  In pair
      // mode the leader's barriers also count the peer's copies.
      // A drain that runs out is recorded like any other timeout: the copy may
      // still land after the CTA has exited, so nothing the grid produced (nor
      // anything later on this context) can be trusted.
      for (int s = 0; s < STAGES; ++s)
        if ((issued_mask & (1u << s)) && !mbar_drain(&ctl->full[s], (issued_phase >> s) & 1u, budget))
          record_timeout(p, abort_flag, 0x600u | static_cast<unsigned int>(s));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      const uint32_t IDESC = idesc_f32(Cfg::TILE_M, BN, A_MN, B_MN, p.f16_ops ? FMT_F16 : FMT_BF16);
      constexpr uint32_t IDESC8 = idesc_f32(Cfg::TILE_M, BN, A_MN, B_MN, FMT_E4M3);
      constexpr uint16_t PAIR_MASK = 0x3;
      int stage = 0;
      uint32_t phase = 0, unit = 0;
      bool ok = true;
      for (int w = cluster_id; ok && w < p.num_work; w += num_clusters) {
        const WorkItem it = work_item(w, p, kb_per_unit);
        for (int s = it.s_begin; ok && s < it.s_end; ++s, ++unit) {
          const uint32_t acc = unit % ACCS, acc_phase = (unit / ACCS) & 1u;
          if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, abort_flag, budget)) {
            record_timeout(p, abort_flag, 0x200u);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + acc * BN;  // ACCS == 1: widths at columns 0 and 256
          for (int i = it.i_begin; i < it.i_end; ++i) {
            if (!mbar_wait(&ctl->full[stage], phase, abort_flag, budget)) {
              record_timeout(p, abort_flag, 0x300u);
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t a_base = smem_u32(sA + stage * Cfg::A_BYTES);
            const uint32_t b_base = smem_u32(sB + stage * Cfg::B_STAGE_BYTES);
            if (F8LO && i >= p.kblocks_per_shard) {
              // e4m3 stage: 128 K rows of 128 bytes; each MMA takes K = 32
              // rows (4 groups of 8, 4096 bytes); 128-row MN blocks are one
              // 16 KB box apart
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ad = smem_desc_sw128(a_base + k * 4096, F8_BOX_BYTES, 1024);
#pragma unroll
                for (int w = 0; w < Cfg::WIDTHS; ++w) {
                  const uint64_t bd = smem_desc_sw128(b_base + w * Cfg::SUB_BYTES + k * 4096, F8_BOX_BYTES, 1024);
                  const uint32_t accumulate = (i != it.i_begin || k != 0) ? 1u : 0u;
                  if constexpr (PAIR) {
                    mma_f8_pair(d_tmem + w * BN, ad, bd, IDESC8, accumulate);
                  } else {
                    mma_f8_ss(d_tmem + w * BN, ad, bd, IDESC8, accumulate);
                  }
                }
              }
            } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              // K-major: the 16-wide K slice is 32 bytes further along each
              // 128-byte swizzled row; 8-row groups are 1024 bytes apart.
              // MN-major: the slice is 16 rows (2 groups of 8, 2048 bytes)
              // further; 64-wide MN blocks are one 8 KB box apart.
              const uint64_t ad = A_MN ? smem_desc_sw128(a_base + k * 2048, MN_BOX_BYTES, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
#pragma unroll
              for (int w = 0; w < Cfg::WIDTHS; ++w) {
                const uint32_t bw = b_base + w * Cfg::SUB_BYTES;
                const uint64_t bd = B_MN ? smem_desc_sw128(bw + k * 2048, MN_BOX_BYTES, 1024)
                                         : smem_desc_sw128(bw + k * 32, 16, 1024);
                const uint32_t accumulate = (i != it.i_begin || k != 0) ? 1u : 0u;
                if constexpr (PAIR) {
                  mma_bf16_pair(d_tmem + w * BN, ad, bd, IDESC, accumulate);
                  if constexpr (DUAL) {  // the low half of A into the same accumulator
                    const uint32_t alo = a_base + A_STAGE_BYTES;
                    const uint64_t ad_lo = A_MN ? smem_desc_sw128(alo + k * 2048, MN_BOX_BYTES, 1024)
                                                : smem_desc_sw128(alo + k * 32, 16, 1024);
                    mma_bf16_pair(d_tmem + w * BN, ad_lo, bd, IDESC, 1u);
                  }
                } else {
                  mma_bf16_ss(d_tmem + w * BN, ad, bd, IDESC, accumulate);
                }
              }
            }
            }
            if constexpr (PAIR) {
              mma_commit_pair_multicast(&ctl->empty[stage], PAIR_MASK);
            } else {
              mma_commit(&ctl->empty[stage]);
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          if constexpr (PAIR) {
            mma_commit_pair_multicast(&ctl->tfull[acc], PAIR_MASK);
          } else {
            mma_commit(&ctl->tfull[acc]);
          }
        }
      }
      // Every MMA this thread issued must finish before TMEM is released.
      if constexpr (PAIR) {
        mma_commit_pair(&ctl->mma_done);
      } else {
        mma_commit(&ctl->mma_done);
      }
      if (!mbar_drain(&ctl->mma_done, 0u, budget)) record_timeout(p, abort_flag, 0x700u);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;     // TMEM lane quadrant this warp may access
    const int slice = ew >> 2;  // column slice of the tile (SLICE_COLS columns)
    constexpr int SLICE_COLS = Cfg::SLICE_COLS;
    // the MMA issuer's "accumulator drained" barriers (in the leader CTA)
    // this warp's staging tiles: [fp32 (EPI_BIAS_GELU)] [bf16 out0] [bf16 out1]
    const uint32_t stage_base = smem_u32(sEpi + ew * epi_warp_bytes(EPI));
    const uint32_t st_f32 = stage_base;
    const uint32_t st_out0 = stage_base + (EPI == EPI_BIAS_GELU ? EPI_F32_TILE : 0);
    const uint32_t st_out1 = st_out0 + EPI_BF16_TILE;
    // fp16 + e4m3 mode: the factor that undoes the operands' scales, and the
    // scale of dH (EPI_GELU_GRAD)
    const float out_mul = out_factor(p);
    const float s_dh = p.fp8_stats != nullptr ? fp8_scales(p.fp8_stats).sH : 1.0f;
    uint32_t tempty_addr[2] = {0u, 0u};
    if constexpr (PAIR) {
#pragma unroll
      for (int a = 0; a < ACCS; ++a) tempty_addr[a] = map_shared_to_cta(smem_u32(&ctl->tempty[a]), 0u);
    }
    uint32_t unit = 0;
    bool ok = true;
    for (int w = cluster_id; ok && w < p.num_work; w += num_clusters) {
      const WorkItem it = work_item(w, p, kb_per_unit);
      int mb, nb;
      tile_coords(it.tile, p, mb, nb);
      const int row_block = mb * Cfg::CTAS + static_cast<int>(rank);  // this CTA's 128-row block
      const int row0 = row_block * BM + q * 32;  // this warp's first row
      const int row = row0 + lane;
      const bool row_ok = row < p.M;
      float sum[EPI == EPI_SHARD_SUM ? SLICE_COLS : 1];
      // EPI_PEER: the rank that owns this CTA's 128 token rows, the block's
      // index in that rank's buffers, and (with flags) the wait for the
      // owner to have consumed the previous exchange's values in this slot
      int peer_owner = 0, peer_lb = 0;
      bool peer_blk = false;
      if constexpr (EPI == EPI_PEER) {
        peer_blk = row_block * BM < p.M;
        if (peer_blk) {
          peer_owner = p.peer.world == 1 ? 0 : (row_block * BM) / p.peer.rows;
          peer_lb = row_block - peer_owner * (p.peer.rows / BM);
          if (p.peer.epoch != 0u) {
            if (lane == 0 &&
                !peer_wait_at_least(peer_consumed(p.peer, peer_owner, peer_lb, nb), p.peer.epoch - 1u, budget))
              record_timeout(p, abort_flag, 0x800u);
            __syncwarp();
            if (*abort_flag) {
              ok = false;
              break;
            }
          }
        }
      }
      for (int s = it.s_begin; s < it.s_end; ++s, ++unit) {
        const uint32_t acc = unit % ACCS, acc_phase = (unit / ACCS) & 1u;
        // bias+GeLU on wide tiles (single accumulator, epilogue not hidden):
        // the first chunk's bias is fetched while the mainloop runs, each
        // later chunk's during the chunk before it
        constexpr bool BIAS_AHEAD = EPI == EPI_BIAS_GELU && TN == 512;
        uint4 bias_raw[BIAS_AHEAD ? 4 : 1];
        if constexpr (BIAS_AHEAD) {
          const int col0 = nb * Cfg::TILE_N + slice * SLICE_COLS;
          if (col0 < p.N) load_bf16x32_raw(p.bias + col0, bias_raw);
        }
        if (!mbar_wait(&ctl->tfull[acc], acc_phase, abort_flag, budget)) {
          record_timeout(p, abort_flag, 0x400u);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t t_addr =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + slice * SLICE_COLS;
#pragma unroll
        for (int c = 0; c < SLICE_COLS / 32; ++c) {
          const int col = nb * Cfg::TILE_N + slice * SLICE_COLS + c * 32;
          if (col >= p.N) continue;  // warp-uniform: ragged last column block
          uint32_t r[32];
          tmem_load_32cols(t_addr + c * 32, r);
          // the staging tiles are free again once this warp's previous bulk
          // stores have read them
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          if constexpr (EPI == EPI_BIAS_GELU) {
            // Z = X·A + a (fp32, saved), H = g(Z) saved as (hi, lo)
            float bias[32];
            if constexpr (BIAS_AHEAD) {
              widen_bf16x32(bias_raw, bias);
              if (c + 1 < SLICE_COLS / 32 && col + 32 < p.N) load_bf16x32_raw(p.bias + col + 32, bias_raw);
            } else {
              load_bf16x32(p.bias + col, bias);
            }
            float z[32];
            uint32_t hp[16], lp[16];
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = __uint_as_float(r[j]) + bias[j];
            if (p.fp8_out) {
              // H as fp16 plus its e4m3 residual (H − fp16(H))·2^7
              float big = 0.0f;  // max |H| of the chunk
#pragma unroll
              for (int j = 0; j < 8; ++j) lp[j] = 0u;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float g0 = gelu_f(z[2 * j]), g1 = gelu_f(z[2 * j + 1]);
                big = fmaxf(big, fmaxf(fabsf(g0), fabsf(g1)));
                uint32_t lo8;
                split_f16_e4m3(g0, g1, hp[j], lo8);
                lp[j >> 1] |= lo8 << (16 * (j & 1));
              }
              record_range(p, big >= FP8_H_LIMIT, 0xB01u);
              stage_f32x32(st_f32, lane, z);
              stage_bf16x32(st_out0, lane, hp);  // fp16: same 64-byte rows and swizzle
              stage_e4m3x32(st_out1, lane, reinterpret_cast<const uint32_t(&)[8]>(lp));
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) split_bf16x2(gelu_f(z[2 * j]), gelu_f(z[2 * j + 1]), hp[j], lp[j]);
              stage_f32x32(st_f32, lane, z);
              stage_bf16x32(st_out0, lane, hp);
              stage_bf16x32(st_out1, lane, lp);
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out[2], st_f32, col, row0);
              tma_store_2d(&maps.out[0], st_out0, col, row0);
              tma_store_2d(&maps.out[1], st_out1, col, row0);
              bulk_commit_group();
            }
          } else if constexpr (EPI == EPI_GELU_GRAD) {
            // dH = (dY·Bᵀ) ⊙ g'(Z), saved as (hi, lo); fp32 column sums for da
            float z[32];
            load_rows_f32x32_coalesced(p.aux, p.M, p.N, row0, col, stage_base, lane, z);
            float dh[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) dh[j] = row_ok ? __uint_as_float(r[j]) * gelu_grad_f(z[j]) : 0.0f;
            uint32_t hp[16], lp[16];
            if (p.fp8_out) {
              // dH·sH as fp16 plus its e4m3 residual
              float big = 0.0f;  // max |dH·sH| of the chunk
#pragma unroll
              for (int j = 0; j < 8; ++j) lp[j] = 0u;
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float d0 = dh[2 * j] * s_dh, d1 = dh[2 * j + 1] * s_dh;
                big = fmaxf(big, fmaxf(fabsf(d0), fabsf(d1)));
                uint32_t lo8;
                split_f16_e4m3(d0, d1, hp[j], lo8);
                lp[j >> 1] |= lo8 << (16 * (j & 1));
              }
              record_range(p, big >= FP8_H_LIMIT, 0xB02u);
              stage_bf16x32(st_out0, lane, hp);
              stage_e4m3x32(st_out1, lane, reinterpret_cast<const uint32_t(&)[8]>(lp));
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) split_bf16x2(dh[2 * j], dh[2 * j + 1], hp[j], lp[j]);
              stage_bf16x32(st_out0, lane, hp);
              stage_bf16x32(st_out1, lane, lp);
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out[0], st_out0, col, row0);
              tma_store_2d(&maps.out[1], st_out1, col, row0);
              bulk_commit_group();
            }
            if (p.colsum != nullptr) {
              const float cs = warp_column_sums(dh);
              const long long ci = static_cast<long long>(row_block * 4 + q) * p.N + col + lane;
              if (index_ok(ci, p.colsum_elems, p.status, 0x501u)) p.colsum[ci] = cs;
            }
          } else if constexpr (EPI == EPI_PEER) {
            // this warp's 32 rows x 32 columns of the fp32 partial, into
            // slot `rank` of the owner's receive buffer: transposed through
            // the staging tile so 8 lanes write each 128-byte row segment
            if (peer_blk) {
              float v[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * out_mul;  // 1 outside the fp8 mode
              stage_f32x32(st_f32, lane, v);
              __syncwarp();
              const long long base =
                  (static_cast<long long>(p.peer.rank) * p.peer.rows + (row0 - peer_owner * p.peer.rows)) * p.N + col;
              float* dst = p.peer.recv[peer_owner];
              const int rr = lane >> 3, cc = lane & 7;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int rw = i * 4 + rr;
                const long long di = base + static_cast<long long>(rw) * p.N + cc * 4;
                if (row0 + rw < p.M && index_ok(di + 3, p.peer_recv_elems, p.status, 0x509u))
                  st_global_v4f(dst + di, ld_shared_v4f(st_f32 + rw * 128 + ((cc ^ (rw & 7)) << 4)));
              }
              __syncwarp();
            }
          } else if constexpr (EPI == EPI_STORE) {
            if (it.piece >= 0) {
              // one K piece of a split tile: its fp32 sum goes to the scratch
              const long long si = static_cast<long long>(it.piece) * (Cfg::TILE_M * Cfg::TILE_N) +
                                   static_cast<long long>(rank * BM + q * 32 + lane) * Cfg::TILE_N + slice * SLICE_COLS +
                                   c * 32;
              if (!index_ok(si + 31, p.scratch_elems, p.status, 0x502u)) continue;
              float4* d4 = reinterpret_cast<float4*>(p.tail_scratch + si);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                    __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
              continue;
            }
            uint32_t op[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              op[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * out_mul, __uint_as_float(r[2 * j + 1]) * out_mul);
            stage_bf16x32(st_out0, lane, op);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out[0], st_out0, col, row0);
              bulk_commit_group();
            }
          } else {  // EPI_SHARD_SUM
            if (s == it.s_begin) {
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[c * 32 + j] = __uint_as_float(r[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[c * 32 + j] += __uint_as_float(r[j]);
            }
            if (s == it.s_end - 1 && it.piece >= 0) {
              // one piece of a split tile: its fp32 sum goes to the scratch
              const long long si = static_cast<long long>(it.piece) * (Cfg::TILE_M * Cfg::TILE_N) +
                                   static_cast<long long>(rank * BM + q * 32 + lane) * Cfg::TILE_N + slice * SLICE_COLS +
                                   c * 32;
              if (index_ok(si + 31, p.scratch_elems, p.status, 0x503u)) {
                float4* d4 = reinterpret_cast<float4*>(p.tail_scratch + si);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  d4[j] = make_float4(sum[c * 32 + 4 * j], sum[c * 32 + 4 * j + 1], sum[c * 32 + 4 * j + 2],
                                      sum[c * 32 + 4 * j + 3]);
              }
            } else if (s == it.s_end - 1) {
              // 8 columns at a time (one 16-byte bias load, one 16-byte
              // staging store), so few values beyond the running sums are live
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const uint4 braw = p.bias != nullptr ? __ldg(reinterpret_cast<const uint4*>(p.bias + col) + g)
                                                     : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
                uint32_t yp[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 bv = unpack_bf16x2(bw[e]);
                  yp[e] = pack_bf16x2(fmaf(sum[c * 32 + 8 * g + 2 * e], out_mul, bv.x),
                                      fmaf(sum[c * 32 + 8 * g + 2 * e + 1], out_mul, bv.y));
                }
                st_shared_v4(st_out0 + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4), yp[0], yp[1], yp[2], yp[3]);
              }
              fence_proxy_async_shared();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&maps.out[0], st_out0, col, row0);
                bulk_commit_group();
              }
            }
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) {
            mbar_arrive_cluster(tempty_addr[acc]);
          } else {
            mbar_arrive(&ctl->tempty[acc]);
          }
        }
      }
      if constexpr (EPI == EPI_PEER) {
        // every lane's stores reach the owner before this warp's arrival does
        if (ok && peer_blk && p.peer.epoch != 0u) {
          __threadfence_system();
          __syncwarp();
          if (lane == 0) red_add_release_sys(peer_counter(p.peer, peer_owner, peer_lb, nb), 1u);
        }
      }
    }
    // every bulk store this warp issued has completed before the CTA exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // Both CTAs of a pair stay resident until all remote arrivals and
  // multicast commits addressed to them have landed.
  tc_fence_before_sync();
  if constexpr (PAIR) {
    cluster_sync_all();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    if constexpr (PAIR) {
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    } else {
      tmem_dealloc(tmem_base, TMEM_COLS);
    }
  }
}

// Finishes split tiles: out[row, col] = bf16(((piece_0 + piece_1) + ...) +
// bias[col]) over the pieces of each split tile in order (ascending shards or
// ascending K).  Split tiles are [first_tile, first_tile + tiles) with
// `split` pieces each, stored in that order.  One thread per 8 consecutive
// columns of one row of one split tile.
template <int TILE_M, int TILE_N>
__global__ void __launch_bounds__(256) split_reduce_kernel(const GemmParams p, int first_tile, int tiles, int split) {
  grid_wait_prerequisites();  // programmatic dependent launch, as the GEMMs
  grid_launch_dependents();
  constexpr int COLS8 = TILE_N / 8;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(tiles) * TILE_M * COLS8) return;
  const int t_local = static_cast<int>(idx / (TILE_M * COLS8));
  const int rem = static_cast<int>(idx % (TILE_M * COLS8));
  const int r = rem / COLS8, c8 = (rem % COLS8) * 8;
  int mb, nb;
  tile_coords(first_tile + t_local, p, mb, nb);
  const int row = mb * TILE_M + r, col = nb * TILE_N + c8;
  if (row >= p.M || col >= p.N) return;
  float acc[8];
  for (int part = 0; part < split; ++part) {
    const long long si = static_cast<long long>(t_local * split + part) * (TILE_M * TILE_N) +
                         static_cast<long long>(r) * TILE_N + c8;
    if (!index_ok(si + 7, p.scratch_elems, p.status, 0x504u)) return;
    const float4* src = reinterpret_cast<const float4*>(p.tail_scratch + si);
    const float4 v0 = src[0], v1 = src[1];
    const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = part == 0 ? v[e] : acc[e] + v[e];
  }
  const float mul = out_factor(p);
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= mul;
  float bias[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) bias[e] = 0.0f;
  if (p.bias != nullptr) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(u[e]);
      bias[2 * e] = f.x;
      bias[2 * e + 1] = f.y;
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0] + bias[0], acc[1] + bias[1]);
  o.y = pack_bf16x2(acc[2] + bias[2], acc[3] + bias[3]);
  o.z = pack_bf16x2(acc[4] + bias[4], acc[5] + bias[5]);
  o.w = pack_bf16x2(acc[6] + bias[6], acc[7] + bias[7]);
  const long long oi = static_cast<long long>(row) * p.N + col;
  if (index_ok(oi + 7, static_cast<long long>(p.M) * p.N, p.status, 0x505u))
    *reinterpret_cast<uint4*>(p.out0 + oi) = o;
}

}  // namespace mlptp
