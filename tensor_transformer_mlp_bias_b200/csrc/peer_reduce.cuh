// The owner's side of the cross-GPU shard reduction (peer.cuh): the sum of
// the `world` fp32 partials of this rank's token rows, in rank order, plus
// the bias, rounded once to bf16.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "gemm.cuh"  // index_ok, status codes
#include "peer.cuh"

namespace mlptp {

constexpr int PEER_ROWS_IN_FLIGHT = 4;  // rows of loads each thread keeps in flight

// The owner's side: one CTA of 256 threads per (128-row block, 256-column
// block) of this rank's token rows.  Thread x of 64 owns 4 consecutive
// columns; the 4 row phases walk the block's rows.
__global__ void __launch_bounds__(256, 4) peer_reduce_kernel(const PeerParams q, const __nv_bfloat16* __restrict__ bias,
                                                          int N, __nv_bfloat16* __restrict__ out, unsigned int* status,
                                                          unsigned long long budget_ns, long long recv_elems) {
  grid_wait_prerequisites();  // programmatic dependent launch, as the GEMMs
  grid_launch_dependents();
  const int lb = static_cast<int>(blockIdx.x) / q.ncb;
  const int cb = static_cast<int>(blockIdx.x) % q.ncb;
  __shared__ int go;
  if (threadIdx.x == 0) {
    bool ok = true;
    if (q.epoch != 0u)
      ok = peer_wait_at_least(peer_counter(q, q.rank, lb, cb),
                              q.epoch * static_cast<unsigned int>(q.world) * static_cast<unsigned int>(PEER_ARRIVALS),
                              budget_ns);
    if (!ok) {
      atomicCAS(status, 0u, STATUS_TIMEOUT);
      atomicCAS(status + 1, 0u, 0x900u);
    }
    go = ok ? 1 : 0;
  }
  __syncthreads();
  if (!go) return;
  const float* recv = q.recv[q.rank];
  const int col = cb * PEER_BLOCK_COLS + (static_cast<int>(threadIdx.x) & 63) * 4;
  if (col < N) {
    float b[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (bias != nullptr) {
      const uint2 w = *reinterpret_cast<const uint2*>(bias + col);
      const __nv_bfloat162 b01 = *reinterpret_cast<const __nv_bfloat162*>(&w.x);
      const __nv_bfloat162 b23 = *reinterpret_cast<const __nv_bfloat162*>(&w.y);
      b[0] = __low2float(b01);
      b[1] = __high2float(b01);
      b[2] = __low2float(b23);
      b[3] = __high2float(b23);
    }
    const size_t slot = static_cast<size_t>(q.rows) * static_cast<size_t>(N);
    // PEER_ROWS_IN_FLIGHT rows per thread per pass (4 row phases), every
    // slot's loads issued before the sums use them; few enough registers that
    // the grid (one CTA per block) fits one wave
    constexpr int RIF = PEER_ROWS_IN_FLIGHT;
    const int rows_here = min(PEER_BLOCK_ROWS, q.rows - lb * PEER_BLOCK_ROWS);
    const size_t step = static_cast<size_t>(4) * static_cast<size_t>(N);
    for (int r0 = static_cast<int>(threadIdx.x) >> 6; r0 < rows_here; r0 += 4 * RIF) {
      const size_t off0 = static_cast<size_t>(lb * PEER_BLOCK_ROWS + r0) * static_cast<size_t>(N) + col;
      const int live = min(RIF, (rows_here - r0 + 3) / 4);  // rows r0, r0+4, ... below rows_here
      if (!index_ok(static_cast<long long>((q.world - 1) * slot + off0 + (live - 1) * step + 3), recv_elems, status,
                    0x50au))
        break;
      float4 acc[RIF];
#pragma unroll
      for (int j = 0; j < RIF; ++j)
        acc[j] = j < live ? __ldcg(reinterpret_cast<const float4*>(recv + off0 + j * step)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
      for (int s = 1; s < q.world; ++s) {  // rank order
        const float* src = recv + s * slot + off0;
        float4 v[RIF];
#pragma unroll
        for (int j = 0; j < RIF; ++j)
          v[j] = j < live ? __ldcg(reinterpret_cast<const float4*>(src + j * step)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < RIF; ++j) {
          acc[j].x += v[j].x;
          acc[j].y += v[j].y;
          acc[j].z += v[j].z;
          acc[j].w += v[j].w;
        }
      }
#pragma unroll
      for (int j = 0; j < RIF; ++j) {
        if (j >= live) continue;
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x + b[0], acc[j].y + b[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z + b[2], acc[j].w + b[3]);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&lo);
        o.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + off0 + j * step) = o;
      }
    }
  }
  if (q.epoch != 0u) {
    // every read of the slots above is done before the writers may reuse them
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence_system();
      st_release_sys(peer_consumed(q, q.rank, lb, cb), q.epoch);
    }
  }
}

}  // namespace mlptp
