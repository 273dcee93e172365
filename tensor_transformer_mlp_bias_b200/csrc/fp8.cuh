// The fp16 + e4m3 precision mode (MLP_TP_FP8): operand copies, their scales
// and the packing helpers the GEMM epilogues use.
//
// A product that needs more than bf16's 8 significant bits runs as an fp16
// product (11 bits) plus an 8-bit residual product in the same fp32
// accumulator:
//   dB = Hᵀ·dY:  H16 = fp16(H),  H8 = e4m3((H − H16)·2^7)
//                dY16 = fp16(dY·sY),  dY8 = e4m3(dY·sY·2^-7)
//                dB = (H16ᵀ·dY16 + H8ᵀ·dY8) / sY
//   dA = Xᵀ·dH:  X16 = fp16(X·sX),  X8 = e4m3(X·sX·2^-7)
//                dH16 = fp16(dH·sH),  dH8 = e4m3((dH·sH − dH16)·2^7)
//                dA = (X16ᵀ·dH16 + X8ᵀ·dH8) / (sX·sH)
// The 2^7 and 2^-7 cancel in each residual product, so both products carry
// the same scale.  Y and dX take one fp16 product each (H16 with an fp16 copy
// of B, dH16 with an fp16 copy of A).  The residual term is about 2^-11 of
// its product and keeps 4 significant bits, so each weight gradient keeps
// about 15 bits, at 1.5 bf16-products of tensor time instead of the 2 of the
// bf16 pair.
//
// Scales are powers of two (exact to apply and to undo):
//   sX, sY  largest power of two with max|X|·sX (max|dY|·sY) <= 2^15, so
//           the fp16 copy cannot overflow and the e4m3 copy stays below 2^8;
//   sH      largest power of two with bound·sH <= 2^12, where
//           bound = 1.212·max_t‖dY_t‖·max_k‖B_k‖ >= max|dH|
//           (|dH| <= max|g'|·|dY_t·B_k| and Cauchy–Schwarz; max|g'| < 1.2;
//           1.01 covers the fp32 sums of squares), so |dH·sH| < 2^13 and the
//           residual e4m3((dH·sH − dH16)·2^7) cannot saturate.
//   H       unscaled: the residual saturates only for |H| >= 2^13, which the
//           epilogue records as MLP_ERR_RANGE.
// The statistics (max|X|, max|dY|, the two largest squared row norms) are
// reduced by fp8_stats_kernel into four words of the workspace header; every
// consumer derives the scales from them with the same function.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"

namespace mlptp {

constexpr unsigned int STATUS_RANGE = 9u;
constexpr float FP8_LO_SHIFT = 128.0f;        // 2^7 between a residual and its partner
constexpr float FP8_H_LIMIT = 8192.0f;        // |H|, |dH·sH| below this: the residual fits e4m3
constexpr float FP16_MAX = 65504.0f;

// Word offsets of the statistics in the workspace header (float bits, >= 0,
// combined with atomicMax): max|X|, max|dY|, max_t ‖dY_t‖², max_k ‖B_k‖².
enum Fp8Stat : int { STAT_AMAX_X = 0, STAT_AMAX_DY = 1, STAT_SS_DY = 2, STAT_SS_B = 3, STAT_WORDS = 4 };

// Largest power of two s with v·s <= 2^e_target, for v >= 0 (1 for v == 0
// or a non-finite v), clamped to [2^-100, 2^100].  Works on the exponent and
// mantissa bits of v, so it is exact.
__device__ __forceinline__ float pow2_scale_below(int e_target, float v) {
  if (!(v > 0.0f)) return 1.0f;
  const uint32_t bits = __float_as_uint(v);
  const int ex = static_cast<int>((bits >> 23) & 0xffu);
  if (ex == 0xff) return 1.0f;
  int k;
  if (ex == 0) {
    k = e_target + 126;  // subnormal v < 2^-126
  } else {
    const bool pow2 = (bits & 0x7fffffu) == 0u;
    k = e_target - (ex - 127) - (pow2 ? 0 : 1);
  }
  k = k < -100 ? -100 : (k > 100 ? 100 : k);
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

struct Fp8Scales {
  float sX, sY, sH;
};

__device__ __forceinline__ Fp8Scales fp8_scales(const unsigned int* stats) {
  Fp8Scales s;
  s.sX = pow2_scale_below(15, __uint_as_float(stats[STAT_AMAX_X]));
  s.sY = pow2_scale_below(15, __uint_as_float(stats[STAT_AMAX_DY]));
  const float bound = 1.212f * sqrtf(__uint_as_float(stats[STAT_SS_DY])) * sqrtf(__uint_as_float(stats[STAT_SS_B]));
  s.sH = pow2_scale_below(12, bound);
  return s;
}

// (lo, hi) -> fp16x2 bits, lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<__half2*>(&v));
}

// Two values -> e4m3x2 bits (round to nearest, saturating), v0 in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float v0, float v1) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(v0, v1), __NV_SATFINITE, __NV_E4M3));
}

// v0, v1 -> fp16 pair `hi` and the e4m3 residuals (v - fp16(v))·2^7, packed
// into 16 bits `lo8` (v0 in the low byte).
__device__ __forceinline__ void split_f16_e4m3(float v0, float v1, uint32_t& hi, uint32_t& lo8) {
  hi = pack_f16x2(v0, v1);
  const float2 h = unpack_f16x2(hi);
  lo8 = pack_e4m3x2((v0 - h.x) * FP8_LO_SHIFT, (v1 - h.y) * FP8_LO_SHIFT);
}

// Row `r` (this lane) of a 32x32 e4m3 staging tile: 32-byte rows, 16-byte
// chunk j stored at chunk j ^ ((r >> 2) & 1) (the TMA 32-byte swizzle; the
// tile is 256-byte aligned), so a warp's 16-byte stores hit every bank.
__device__ __forceinline__ void stage_e4m3x32(uint32_t tile, int r, const uint32_t (&packed)[8]) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
    st_shared_v4(tile + r * 32 + ((j ^ ((r >> 2) & 1)) << 4), packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                 packed[4 * j + 3]);
}

// ---------------------------------------------------------------- statistics
// Rows of length h from three bf16 matrices: X[T,h] (max|x|), dY[T,h]
// (max|x| and the largest row sum of squares), B[f,h] (largest row sum of
// squares).  One warp per row at a time; each block combines its warps and
// raises the four words once.  The words must be zero before the launch.
constexpr int STATS_THREADS = 256;

__device__ __forceinline__ void atomic_max_nonneg(unsigned int* word, float v) {
  atomicMax(word, __float_as_uint(v));  // non-negative floats order like their bits
}

__global__ void __launch_bounds__(STATS_THREADS) fp8_stats_kernel(const __nv_bfloat16* X, const __nv_bfloat16* dY,
                                                                  const __nv_bfloat16* B, int T, int h, int f,
                                                                  unsigned int* stats) {
  grid_wait_prerequisites();
  grid_launch_dependents();
  constexpr int WARPS = STATS_THREADS / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float amax_x = 0.0f, amax_dy = 0.0f, ss_dy = 0.0f, ss_b = 0.0f;
  const long long rows = 2LL * T + f;
  for (long long r = static_cast<long long>(blockIdx.x) * WARPS + warp; r < rows;
       r += static_cast<long long>(gridDim.x) * WARPS) {
    const int which = r < T ? 0 : (r < 2LL * T ? 1 : 2);
    const long long row = which == 0 ? r : (which == 1 ? r - T : r - 2LL * T);
    const __nv_bfloat16* src = (which == 0 ? X : (which == 1 ? dY : B)) + row * h;
    float mx = 0.0f, ss = 0.0f;
#pragma unroll 4
    for (int c = lane * 8; c < h; c += 256) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + c));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
        mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, ss));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    if (which == 0) {
      amax_x = fmaxf(amax_x, mx);
    } else if (which == 1) {
      amax_dy = fmaxf(amax_dy, mx);
      ss_dy = fmaxf(ss_dy, ss);
    } else {
      ss_b = fmaxf(ss_b, ss);
    }
  }
  __shared__ float red[WARPS][STAT_WORDS];
  if (lane == 0) {
    red[warp][STAT_AMAX_X] = amax_x;
    red[warp][STAT_AMAX_DY] = amax_dy;
    red[warp][STAT_SS_DY] = ss_dy;
    red[warp][STAT_SS_B] = ss_b;
  }
  __syncthreads();
  if (threadIdx.x < STAT_WORDS) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    if (m > 0.0f) atomic_max_nonneg(stats + threadIdx.x, m);
  }
}

// ---------------------------------------------------------------- casts
// Up to three element-wise jobs, one after the other over the whole grid,
// 8 elements per thread and step: dst16 = fp16(src·s) and, when dst8 is not
// NULL, dst8 = e4m3(src·s·2^-7).  s = 1 (weights; a value that fp16 cannot
// hold records MLP_ERR_RANGE), sX or sY.
enum CastScale : int { CAST_UNSCALED = 0, CAST_SX = 1, CAST_SY = 2 };
struct CastJob {
  const __nv_bfloat16* src;
  __half* dst16;
  uint8_t* dst8;
  long long n;  // elements, a multiple of 8
  int scale;
};
struct CastJobs {
  CastJob job[3];
  int count;
};

constexpr int CAST_UNROLL = 4;  // 16-byte loads in flight per thread

__device__ __forceinline__ void cast_group(const uint4 w, const CastJob& jb, float s, float s8, long long g,
                                           bool& bad) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  uint32_t o16[4], o8[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
    if (jb.scale == CAST_UNSCALED) bad |= fabsf(v.x) > FP16_MAX || fabsf(v.y) > FP16_MAX;
    o16[e] = pack_f16x2(v.x * s, v.y * s);
    o8[e >> 1] |= pack_e4m3x2(v.x * s8, v.y * s8) << (16 * (e & 1));
  }
  reinterpret_cast<uint4*>(jb.dst16)[g] = make_uint4(o16[0], o16[1], o16[2], o16[3]);
  if (jb.dst8 != nullptr) reinterpret_cast<uint2*>(jb.dst8)[g] = make_uint2(o8[0], o8[1]);
}

__global__ void __launch_bounds__(256) fp8_cast_kernel(const __grid_constant__ CastJobs jobs, const unsigned int* stats,
                                                       unsigned int* status) {
  grid_wait_prerequisites();
  grid_launch_dependents();
  const Fp8Scales sc = stats != nullptr ? fp8_scales(stats) : Fp8Scales{1.0f, 1.0f, 1.0f};
  bool bad = false;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (int j = 0; j < jobs.count; ++j) {
    const CastJob& jb = jobs.job[j];
    const float s = jb.scale == CAST_SX ? sc.sX : (jb.scale == CAST_SY ? sc.sY : 1.0f);
    const float s8 = s / FP8_LO_SHIFT;
    const long long groups = jb.n / 8;  // 8 values (16 bytes of bf16) per group
    const uint4* src = reinterpret_cast<const uint4*>(jb.src);
    for (long long g0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g0 < groups;
         g0 += CAST_UNROLL * stride) {
      uint4 w[CAST_UNROLL];
#pragma unroll
      for (int q = 0; q < CAST_UNROLL; ++q) {
        const long long g = g0 + q * stride;
        w[q] = g < groups ? __ldg(src + g) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int q = 0; q < CAST_UNROLL; ++q) {
        const long long g = g0 + q * stride;
        if (g < groups) cast_group(w[q], jb, s, s8, g, bad);
      }
    }
  }
  if (bad) {
    atomicCAS(status, 0u, STATUS_RANGE);
    atomicCAS(status + 1, 0u, 0xA00u);
  }
}

}  // namespace mlptp
