// Column sums of a row-major bf16 matrix M[R, C] in fp32, in a fixed order:
// the bias gradients da = Σ_rows dH and db = Σ_rows dY.
//
// Pass 1 (colsum_partial): block (32, COLSUM_PHASES); thread x owns 8
// consecutive columns (one 16-byte load per row, so a warp reads 512
// contiguous bytes of a row); thread y walks rows y, y+PHASES, ... of a chunk
// of ROWS_PER_CHUNK rows.  The row phases are combined through shared memory
// in ascending order and the chunk's partial sums are written to the fp32
// scratch [chunks, C].
// Pass 2 (colsum_final): block (32, 8); thread x owns one column, thread y
// adds the chunk partials y, y+8, ... in ascending order, the 8 phases are
// combined in ascending order, and the sum is rounded once to bf16.  The
// result is therefore deterministic and independent of the launch
// configuration's timing.  Both passes are HBM-bound (R·C·2 bytes read once)
// when R·C is large; at small sizes the row phases supply the loads in
// flight.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "gemm.cuh"  // index_ok, the bounds-checking build's index check

namespace mlptp {

constexpr int COLSUM_ROWS_PER_CHUNK = 256;
constexpr int COLSUM_COLS_PER_BLOCK = 32 * 8;
constexpr int COLSUM_PHASES = 32;  // row phases per block in pass 1

__global__ void __launch_bounds__(32 * COLSUM_PHASES) colsum_partial(const __nv_bfloat16* __restrict__ m, int R,
                                                                     int C, float* __restrict__ partial,
                                                                     long long partial_elems, unsigned int* status) {
  // launched with programmatic dependent launch: every global access below
  // follows the previous grid's completion
  grid_wait_prerequisites();
  grid_launch_dependents();
  __shared__ float red[COLSUM_PHASES][32][9];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int c0 = (blockIdx.x * 32 + tx) * 8;
  const int r_begin = blockIdx.y * COLSUM_ROWS_PER_CHUNK;
  const int r_end = min(R, r_begin + COLSUM_ROWS_PER_CHUNK);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  if (c0 < C) {
    const __nv_bfloat16* base = m + c0;
    for (int r = r_begin + ty; r < r_end; r += COLSUM_PHASES) {
      if (!index_ok(static_cast<long long>(r) * C + c0 + 7, static_cast<long long>(R) * C, status, 0x506u)) break;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * C));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&u[e]);
        const float2 f = __bfloat1622float2(b2);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[ty][tx][e] = acc[e];
  __syncthreads();
  if (ty == 0 && c0 < C) {
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float s = red[0][tx][e];
#pragma unroll
      for (int y = 1; y < COLSUM_PHASES; ++y) s += red[y][tx][e];
      out[e] = s;
    }
    const long long pi = static_cast<long long>(blockIdx.y) * C + c0;
    if (index_ok(pi + 7, partial_elems, status, 0x507u)) {
      float4* dst = reinterpret_cast<float4*>(partial + pi);
      dst[0] = make_float4(out[0], out[1], out[2], out[3]);
      dst[1] = make_float4(out[4], out[5], out[6], out[7]);
    }
  }
}

__global__ void __launch_bounds__(256) colsum_final(const float* __restrict__ partial, int chunks, int C,
                                                    __nv_bfloat16* __restrict__ out, long long partial_elems,
                                                    unsigned int* status) {
  grid_wait_prerequisites();
  grid_launch_dependents();
  __shared__ float red[8][33];
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int c = blockIdx.x * 32 + tx;
  float s = 0.0f;
  if (c < C && index_ok(static_cast<long long>(chunks - 1) * C + c, partial_elems, status, 0x508u)) {
    for (int k = ty; k < chunks; k += 8) s += partial[static_cast<size_t>(k) * C + c];
  }
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && c < C) {
    float t = red[0][tx];
#pragma unroll
    for (int y = 1; y < 8; ++y) t += red[y][tx];
    out[c] = __float2bfloat16_rn(t);
  }
}

}  // namespace mlptp
