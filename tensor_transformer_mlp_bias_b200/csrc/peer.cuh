// The block sharded over `world` GPUs with the shard reduction fused into the
// GEMM epilogue ("Megatron-LM — 架构与原理", §4 巧妙之处: the row-parallel
// layer's outputs are summed once, the forward all-reduce of the reduce
// operator; its backward twin is the copy operator's all-reduce of dX).
//
// Each rank r runs its shard's row-parallel GEMM (P_r = H_r·B_r, or
// Q_r = dH_r·A_rᵀ for dX).  The tokens are split over the ranks (rank o owns
// rows [o·rows, (o+1)·rows)), and the epilogue of every 128-row block of P_r
// stores its fp32 values straight into the owner's receive buffer, slot r,
// over NVLink with plain coalesced stores; no TMA touches peer memory.  The
// owner's reduce kernel then adds the `world` slots in rank order, adds the
// bias once and rounds once to bf16: the reduce-scatter half of the
// all-reduce, with fp32 partials and one rounding.
//
// Receive buffer of rank o:  [world][rows][h] fp32 (slot r from rank r).
// Flag block of rank o:      [nbl][ncb] arrival counters, then [nbl][ncb]
//                            consumed marks (uint32), nbl = ceil(rows/128)
//                            row blocks and ncb = ceil(h/256) column blocks.
//
// Protocol for exchange number `epoch` (1, 2, 3, ... on the same buffers):
//   writer (GEMM epilogue warp of rank r, tile block (lb, cb) owned by o):
//     wait until consumed[o][lb][cb] >= epoch - 1   (the slot is free again)
//     store its 32 rows x 128 columns of fp32 into slot r
//     fence.sys, then counter[o][lb][cb] += 1 (release, system scope)
//   owner (reduce kernel of rank o, one CTA per (lb, cb)):
//     wait until counter[o][lb][cb] >= epoch·world·PEER_ARRIVALS
//     out = bf16(((slot 0 + slot 1) + ...) + bias)
//     consumed[o][lb][cb] = epoch (release, system scope)
// Every wait is bounded; one that runs out records MLP_ERR_TIMEOUT in the
// caller's status word.  Counters only grow, so nothing is reset between
// exchanges.  With epoch == 0 no flag is touched: the caller orders the
// producer and the consumer itself (one stream, or a collective between).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace mlptp {

constexpr int PEER_MAX_WORLD = 8;
constexpr int PEER_BLOCK_ROWS = 128;  // one CTA's rows of a pair tile
constexpr int PEER_BLOCK_COLS = 256;  // one MMA width
constexpr int PEER_ARRIVALS = 8;      // epilogue warps per CTA: 4 lane quadrants x 2 column slices

struct PeerParams {
  float* recv[PEER_MAX_WORLD];          // rank o's receive buffer, as addressed from this GPU
  unsigned int* flags[PEER_MAX_WORLD];  // rank o's flag block, likewise
  int rank, world;
  int rows;          // token rows per rank
  int nbl, ncb;      // 128-row blocks per rank, 256-column blocks
  unsigned int epoch;
};

__device__ __forceinline__ unsigned int* peer_counter(const PeerParams& q, int owner, int lb, int cb) {
  return q.flags[owner] + static_cast<long long>(lb) * q.ncb + cb;
}

__device__ __forceinline__ unsigned int* peer_consumed(const PeerParams& q, int owner, int lb, int cb) {
  return q.flags[owner] + static_cast<long long>(q.nbl) * q.ncb + static_cast<long long>(lb) * q.ncb + cb;
}

// System-scope flag accesses (peer memory over NVLink, or this GPU's own).
__device__ __forceinline__ unsigned int ld_acquire_sys(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_sys(unsigned int* p, unsigned int v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_release_sys(unsigned int* p, unsigned int v) {
  asm volatile("red.release.sys.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_global_v4f(float* p, float4 v) {
  asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

// Bounded wait for *p to reach `target` (modulo 2^32: (int)(*p - target) >= 0).
// Returns false when `budget_ns` of wall time passed first.
__device__ __forceinline__ bool peer_wait_at_least(const unsigned int* p, unsigned int target, uint64_t budget_ns) {
  if (static_cast<int>(ld_acquire_sys(p) - target) >= 0) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (static_cast<int>(ld_acquire_sys(p) - target) >= 0) return true;
    if ((n & 15u) == 0u && global_timer_ns() - t0 > budget_ns) return false;
    __nanosleep(128);
  }
}

}  // namespace mlptp
