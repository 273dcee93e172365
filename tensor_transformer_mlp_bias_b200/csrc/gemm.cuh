// Persistent, warp-specialised tcgen05 GEMM with the MLP block's fused
// epilogues, for sm_100a.
//
//   D[M,N] = sum_k Aop[M,k] · Bop[k,N]   (bf16 in, fp32 accumulate in TMEM)
//
// One CTA per SM walks a static list of 128x256 output tiles.  Warp roles:
//   warp 0      TMA producer: fills a ring of STAGES shared-memory stages
//               (A tile 128x64, B tile 256x64, 128-byte swizzle) and arms a
//               "full" mbarrier with the expected byte count;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators),
//               and one thread issues tcgen05.mma (M=128, N=256, K=16) per
//               16-wide K slice, committing each stage back to its "empty"
//               barrier and each finished accumulator to a "tmem full"
//               barrier;
//   warps 2-9   epilogue: tcgen05.ld the accumulator (one row per thread,
//               32 columns per load), apply the fused math, store bf16 to
//               global memory, release the accumulator.
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
// Operand layouts.  A K-major operand is stored [rows, K] with K contiguous
// and arrives as one TMA box of 64 (K) x rows.  An MN-major operand is
// stored [K, rows] with rows contiguous and arrives as 64-row-wide boxes of
// 64 (rows) x 64 (K); the MMA reads it through an MN-major descriptor, so no
// transpose is ever materialised.
//
// Every wait is bounded (see mbar_wait).  A wait that runs out records
// status 7 (timeout) in the device status word, raises a CTA-wide abort
// flag so the other roles leave their loops, and the CTA still drains its
// in-flight TMA copies and tensor-core operations and frees its TMEM before
// returning.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace mlptp {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int MN_BOX_BYTES = 64 * BK * 2;   // one 64x64 bf16 box, 8 KB
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + NUM_EPI_WARPS * 32;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int CTL_BYTES = 1024;
constexpr int GEMM_SMEM_BYTES = STAGES * STAGE_BYTES + CTL_BYTES + 1024;  // + alignment slack

constexpr unsigned int STATUS_TIMEOUT = 7u;

enum Epi : int { EPI_BIAS_GELU = 0, EPI_SHARD_SUM = 1, EPI_GELU_GRAD = 2, EPI_STORE = 3 };

struct GemmParams {
  int M, N;
  int shards;             // K segments reduced in the epilogue (EPI_SHARD_SUM); 1 otherwise
  int kblocks_per_shard;  // BK-wide K slices per segment
  int m_blocks, n_blocks, num_tiles, group_m;
  __nv_bfloat16* out0;        // Z | Y | dH | dX | dA | dB
  __nv_bfloat16* out1;        // H (EPI_BIAS_GELU)
  const __nv_bfloat16* bias;  // a (EPI_BIAS_GELU) or b (EPI_SHARD_SUM), may be null for the latter
  const __nv_bfloat16* aux;   // Z (EPI_GELU_GRAD)
  unsigned int* status;       // device status word pair in the workspace
  unsigned long long budget_ns;
  unsigned int debug_flags;
};

struct GemmCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
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

// 32 consecutive bf16 values -> fp32 (vectorised 16-byte loads).
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&dst)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 w = __ldg(s + v);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(u[e]);
      dst[v * 8 + 2 * e] = f.x;
      dst[v * 8 + 2 * e + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&packed)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v)
    d[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
}

// ---------------------------------------------------------------- kernel
template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    mlp_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                    const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  GemmCtl* ctl = reinterpret_cast<GemmCtl*>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], NUM_EPI_WARPS);
    }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tma_a);
    prefetch_tensormap(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort;
  const uint64_t budget = p.budget_ns;
  const int total_kb = p.shards * p.kblocks_per_shard;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: filled at least once / parity of last fill
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p, mb, nb);
        const int m0 = mb * BM, n0 = nb * BN;
        for (int kb = 0; kb < total_kb; ++kb) {
          if ((p.debug_flags & 1u) && (tile != (int)blockIdx.x || kb >= 1)) {
            ok = false;  // test hook: stop feeding the tensor core
            break;
          }
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, abort_flag, budget)) {
            record_timeout(p, abort_flag, 0x100u);
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          mbar_arrive_expect_tx(&ctl->full[stage], STAGE_BYTES);
          const int k0 = kb * BK;
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * B_STAGE_BYTES);
          if (A_MN) {
            tma_load_2d(a_dst, &tma_a, fb, m0, k0);
            tma_load_2d(a_dst + MN_BOX_BYTES, &tma_a, fb, m0 + 64, k0);
          } else {
            tma_load_2d(a_dst, &tma_a, fb, k0, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * MN_BOX_BYTES, &tma_b, fb, n0 + 64 * j, k0);
          } else {
            tma_load_2d(b_dst, &tma_b, fb, k0, n0);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // No TMA write may still be landing in this CTA's shared memory when it
      // exits: wait for the last fill of every stage (immediate when the
      // tensor-core warp already consumed it).
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) mbar_drain(&ctl->full[s], (issued_phase >> s) & 1u, budget);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0, unit = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        for (int s = 0; ok && s < p.shards; ++s, ++unit) {
          const uint32_t acc = unit & 1u, acc_phase = (unit >> 1) & 1u;
          if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, abort_flag, budget)) {
            record_timeout(p, abort_flag, 0x200u);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + acc * BN;
          for (int kb = 0; kb < p.kblocks_per_shard; ++kb) {
            if (!mbar_wait(&ctl->full[stage], phase, abort_flag, budget)) {
              record_timeout(p, abort_flag, 0x300u);
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t a_base = smem_u32(sA + stage * A_STAGE_BYTES);
            const uint32_t b_base = smem_u32(sB + stage * B_STAGE_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              // K-major: the 16-wide K slice is 32 bytes further along each
              // 128-byte swizzled row; 8-row groups are 1024 bytes apart.
              // MN-major: the slice is 16 rows (2 groups of 8, 2048 bytes)
              // further; 64-wide MN blocks are one 8 KB box apart.
              const uint64_t ad = A_MN ? smem_desc_sw128(a_base + k * 2048, MN_BOX_BYTES, 1024)
                                       : smem_desc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t bd = B_MN ? smem_desc_sw128(b_base + k * 2048, MN_BOX_BYTES, 1024)
                                       : smem_desc_sw128(b_base + k * 32, 16, 1024);
              mma_bf16_ss(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
            }
            mma_commit(&ctl->empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(&ctl->tfull[acc]);
        }
      }
      // Every MMA this thread issued must finish before TMEM is released.
      mma_commit(&ctl->mma_done);
      mbar_drain(&ctl->mma_done, 0u, budget);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;     // TMEM lane quadrant this warp may access
    const int half = ew >> 2;   // 128-column half of the tile
    uint32_t unit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p, mb, nb);
      const int row = mb * BM + q * 32 + lane;
      const bool row_ok = row < p.M;
      const size_t row_off = static_cast<size_t>(row) * static_cast<size_t>(p.N);
      float sum[EPI == EPI_SHARD_SUM ? 128 : 1];
      for (int s = 0; s < p.shards; ++s, ++unit) {
        const uint32_t acc = unit & 1u, acc_phase = (unit >> 1) & 1u;
        if (!mbar_wait(&ctl->tfull[acc], acc_phase, abort_flag, budget)) {
          record_timeout(p, abort_flag, 0x400u);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t t_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + half * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = nb * BN + half * 128 + c * 32;
          if (col >= p.N) continue;  // warp-uniform: ragged last column block
          uint32_t r[32];
          tmem_load_32cols(t_addr + c * 32, r);
          if constexpr (EPI == EPI_BIAS_GELU) {
            float bias[32];
            load_bf16x32(p.bias + col, bias);
            uint32_t zp[16], hp[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float z0 = __uint_as_float(r[2 * j]) + bias[2 * j];
              const float z1 = __uint_as_float(r[2 * j + 1]) + bias[2 * j + 1];
              zp[j] = pack_bf16x2(z0, z1);
              hp[j] = pack_bf16x2(gelu_f(z0), gelu_f(z1));
            }
            if (row_ok) {
              store_bf16x32(p.out0 + row_off + col, zp);
              store_bf16x32(p.out1 + row_off + col, hp);
            }
          } else if constexpr (EPI == EPI_GELU_GRAD) {
            float z[32];
            if (row_ok) {
              load_bf16x32(p.aux + row_off + col, z);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) z[j] = 0.0f;
            }
            uint32_t dp[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              dp[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * gelu_grad_f(z[2 * j]),
                                  __uint_as_float(r[2 * j + 1]) * gelu_grad_f(z[2 * j + 1]));
            if (row_ok) store_bf16x32(p.out0 + row_off + col, dp);
          } else if constexpr (EPI == EPI_STORE) {
            uint32_t op[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) op[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
            if (row_ok) store_bf16x32(p.out0 + row_off + col, op);
          } else {  // EPI_SHARD_SUM
            if (s == 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[c * 32 + j] = __uint_as_float(r[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[c * 32 + j] += __uint_as_float(r[j]);
            }
            if (s == p.shards - 1) {
              float bias[32];
              if (p.bias != nullptr) {
                load_bf16x32(p.bias + col, bias);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) bias[j] = 0.0f;
              }
              uint32_t yp[16];
#pragma unroll
              for (int j = 0; j < 16; ++j)
                yp[j] = pack_bf16x2(sum[c * 32 + 2 * j] + bias[2 * j], sum[c * 32 + 2 * j + 1] + bias[2 * j + 1]);
              if (row_ok) store_bf16x32(p.out0 + row_off + col, yp);
            }
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace mlptp
