// C-ABI of the tensor-parallel MLP block (declared in include/mlp_tp.h):
// host-side validation, TMA descriptor construction and kernel launches.
// Nothing here allocates device memory or synchronises, except mlp_tp_check.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/mlp_tp.h"
#include "colsum.cuh"
#include "fp8.cuh"
#include "gemm.cuh"
#include "peer_reduce.cuh"

using namespace mlptp;

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_budget_ns{1000000000ull};
std::atomic<uint32_t> g_debug_flags{0};

constexpr size_t WS_HEADER_BYTES = 256;

mlp_status_t fail(mlp_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

mlp_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(MLP_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- shapes
struct Shape {
  int64_t T, h, f;
  int32_t t;
  int64_t fs() const { return f / t; }
};

mlp_status_t check_shape(const Shape& s) {
  if (s.T < 0 || s.h < 0 || s.f < 0) return fail(MLP_ERR_INVALID_ARG, "negative size T=%lld h=%lld f=%lld",
                                                 (long long)s.T, (long long)s.h, (long long)s.f);
  if (s.t < 1) return fail(MLP_ERR_INVALID_ARG, "shard count t=%d must be >= 1", s.t);
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (s.T > lim || s.h > lim || s.f > lim)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "T, h and f must be < 2^31");
  if (s.h < 64 || s.h % 64 != 0) return fail(MLP_ERR_UNSUPPORTED_SHAPE, "h=%lld must be a positive multiple of 64",
                                             (long long)s.h);
  if (s.f % s.t != 0) return fail(MLP_ERR_UNSUPPORTED_SHAPE, "f=%lld is not divisible by t=%d", (long long)s.f, s.t);
  if (s.fs() < 64 || s.fs() % 64 != 0)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "shard width f/t=%lld must be a positive multiple of 64",
                (long long)s.fs());
  return MLP_OK;
}

size_t colsum_chunks(int64_t R) { return static_cast<size_t>((R + COLSUM_ROWS_PER_CHUNK - 1) / COLSUM_ROWS_PER_CHUNK); }
// The GEMMs run on CTA pairs (2-SM tensor-core instructions, 256-row tiles).
#ifndef MLPTP_USE_PAIR
#define MLPTP_USE_PAIR 1
#endif
constexpr bool kPair = MLPTP_USE_PAIR != 0;
// Column tiles.  512 (two MMA widths per CTA pair, one TMEM accumulator)
// reads 25% fewer operand bytes per FLOP from L2, which bounds these GEMMs;
// 256 keeps two accumulators so the epilogue of one tile overlaps the
// mainloop of the next.  Measured on B200: 512 for the weight gradients and
// the bias+GeLU GEMM (its outputs leave through asynchronous TMA stores);
// 256 for the GeLU-derivative GEMM (its epilogue waits on loads of Z) and
// for the shard-sum GEMMs (the running sum of the shard partials is held in
// registers, 128 values per thread at 256 columns).
#ifndef MLPTP_WIDE_TN
#define MLPTP_WIDE_TN 512
#endif
constexpr int kWideTN = kPair ? MLPTP_WIDE_TN : 256;
#ifndef MLPTP_FC1_TN
#define MLPTP_FC1_TN 512
#endif
#ifndef MLPTP_FC2BD_TN
#define MLPTP_FC2BD_TN 256
#endif
constexpr int kFc1TN = kPair ? MLPTP_FC1_TN : 256;    // bias+GeLU GEMM
constexpr int kFc2BdTN = kPair ? MLPTP_FC2BD_TN : 256;  // GeLU-derivative GEMM
#ifndef MLPTP_FC2BD_MANY_WARPS_MAX_K
#define MLPTP_FC2BD_MANY_WARPS_MAX_K 3072
#endif
constexpr int64_t kFc2BdManyWarpsMaxK = MLPTP_FC2BD_MANY_WARPS_MAX_K;
// GEMMs whose A operand is a (hi, lo) pair carry both halves in one stage
// (one pass over K, B read once).
#ifndef MLPTP_DUAL_A
#define MLPTP_DUAL_A 1
#endif
constexpr bool kDualA = kPair && MLPTP_DUAL_A != 0;
using TileShape = TileCfg<kPair, 256, EPI_STORE>;
// 128-row blocks that a GEMM over R rows covers (whole tiles).
size_t gemm_row_blocks(int64_t R) {
  return static_cast<size_t>((R + TileShape::TILE_M - 1) / TileShape::TILE_M) * TileShape::CTAS;
}

// Workspace layout: [status header | dH | dH_lo | fp32 column-sum partials].
size_t pair_bytes(const Shape& s) { return align_up(static_cast<size_t>(s.T * s.f * 2), 256); }
size_t dh_offset() { return WS_HEADER_BYTES; }
size_t dh_lo_offset(const Shape& s) { return WS_HEADER_BYTES + pair_bytes(s); }
size_t partial_offset(const Shape& s) { return WS_HEADER_BYTES + 2 * pair_bytes(s); }
size_t partial_bytes(const Shape& s) {
  // da: one row of column sums per (128-row block, 32-row lane quadrant);
  // db: one row per COLSUM_ROWS_PER_CHUNK rows of dY.
  const size_t da_rows = gemm_row_blocks(s.T) * 4 * static_cast<size_t>(s.f);
  const size_t db_rows = colsum_chunks(s.T) * static_cast<size_t>(s.h);
  return align_up((da_rows > db_rows ? da_rows : db_rows) * sizeof(float), 256);
}
// Pieces of split tiles of the shard-sum GEMMs (outputs [T, h]): at most
// one piece per shard of every tile, and at most TAIL_MAX_PIECES.
constexpr size_t TAIL_MAX_PIECES = 256;
constexpr size_t TAIL_PIECE_BYTES = static_cast<size_t>(TileShape::TILE_M) * BN * sizeof(float);
size_t tail_pieces_capacity(const Shape& s) {
  const size_t tiles = static_cast<size_t>((s.T + TileShape::TILE_M - 1) / TileShape::TILE_M) *
                       static_cast<size_t>((s.h + BN - 1) / BN);
  const size_t n = tiles * static_cast<size_t>(s.t);
  return n < TAIL_MAX_PIECES ? n : TAIL_MAX_PIECES;
}
size_t tail_offset(const Shape& s) { return partial_offset(s) + partial_bytes(s); }
// K pieces of the weight-gradient GEMMs.
//  - Fewer tiles than CTA pairs: at most KSPLIT_MAX_PIECES pieces of 256x512
//    fp32, and no more than one piece per 8 K slices of every tile.
//  - Long token axes: a weight gradient's K loop runs over the T tokens, and
//    one fp32 TMEM accumulator takes at most kWgradMaxAdds tensor-core
//    additions (4 per 64-token K slice and product; both halves of the pair
//    count): 16384 tokens.  Measured on B200: dB over 65536 tokens in one
//    accumulator reached 1.14 of the parity bar, while 16384 tokens pass
//    with a wide margin; the tensor core's accumulation is not round-to-
//    nearest fp32, and its error grows with the number of additions.  Longer
//    K loops are cut into ceil(T / 16384) pieces or more, which the reduce
//    pass adds in fp32 in K order.
constexpr size_t KSPLIT_MAX_PIECES = 128;
constexpr size_t KSPLIT_PIECE_BYTES = static_cast<size_t>(TileShape::TILE_M) * 512 * sizeof(float);
constexpr int64_t kWgradMaxAdds = 2048;
int64_t wgrad_min_pieces(int64_t T) {
  const int64_t adds = 8 * ((T + BK - 1) / BK);  // 4 per slice, times the 2 halves of the pair
  return (adds + kWgradMaxAdds - 1) / kWgradMaxAdds;
}
size_t ksplit_bytes(const Shape& s) {
  const size_t kb = 2 * static_cast<size_t>((s.T + BK - 1) / BK);  // two parts (hi, lo)
  const size_t per_tile = kb / 8;
  const size_t tiles_dA = static_cast<size_t>((s.h + 255) / 256) * static_cast<size_t>((s.f + 511) / 512);
  const size_t tiles_dB = static_cast<size_t>((s.f + 255) / 256) * static_cast<size_t>((s.h + 511) / 512);
  const size_t tiles = tiles_dA > tiles_dB ? tiles_dA : tiles_dB;
  size_t pieces = tiles * per_tile < KSPLIT_MAX_PIECES ? tiles * per_tile : KSPLIT_MAX_PIECES;
  const size_t min_k = static_cast<size_t>(wgrad_min_pieces(s.T));
  if (min_k > 1 && tiles * min_k > pieces) pieces = tiles * min_k;
  return pieces * KSPLIT_PIECE_BYTES;
}
size_t split_scratch_bytes(const Shape& s) {
  const size_t tail = tail_pieces_capacity(s) * TAIL_PIECE_BYTES;
  const size_t ks = ksplit_bytes(s);
  return tail > ks ? tail : ks;
}
size_t workspace_bytes(const Shape& s) { return tail_offset(s) + split_scratch_bytes(s); }

// Recomputation keeps Z, H and H_lo in the workspace after the rest:
// [ ... | Z fp32 | H | H_lo ].
size_t recompute_z_offset(const Shape& s) { return workspace_bytes(s); }
size_t recompute_h_offset(const Shape& s) {
  return recompute_z_offset(s) + align_up(static_cast<size_t>(s.T * s.f * 4), 256);
}
size_t recompute_hlo_offset(const Shape& s) { return recompute_h_offset(s) + pair_bytes(s); }
size_t recompute_workspace_bytes(const Shape& s) { return recompute_hlo_offset(s) + pair_bytes(s); }

// The fp16 + e4m3 mode keeps its operand copies after the rest of the
// workspace: [ ... | W16 (fp16 copy of B in the forward, of A in the
// backward) | X16 | X8 | dY16 | dY8 ], and its statistics in the header.
constexpr size_t FP8_STATS_OFFSET = 64;
struct Fp8Layout {
  size_t w16, x16, x8, dy16, dy8, bytes;
};
Fp8Layout fp8_layout(const Shape& s) {
  Fp8Layout l;
  const size_t th = static_cast<size_t>(s.T * s.h), hf = static_cast<size_t>(s.h * s.f);
  l.w16 = 0;
  l.x16 = l.w16 + align_up(hf * 2, 256);
  l.x8 = l.x16 + align_up(th * 2, 256);
  l.dy16 = l.x8 + align_up(th, 256);
  l.dy8 = l.dy16 + align_up(th * 2, 256);
  l.bytes = l.dy8 + align_up(th, 256);
  return l;
}
size_t mode_workspace_bytes(const Shape& s, int32_t mode, bool recompute) {
  const size_t base = recompute ? recompute_workspace_bytes(s) : workspace_bytes(s);
  return base + (mode == MLP_TP_FP8 ? fp8_layout(s).bytes : 0);
}

struct Ptr {
  const void* p;
  const char* name;
  bool nullable;
  bool empty = false;  // the buffer holds no elements (a T-sized buffer with T == 0): NULL is fine
};

mlp_status_t check_ptrs(std::initializer_list<Ptr> ptrs) {
  for (const Ptr& x : ptrs) {
    if (x.p == nullptr) {
      if (x.nullable || x.empty) continue;
      return fail(MLP_ERR_INVALID_ARG, "pointer %s is NULL", x.name);
    }
    if (reinterpret_cast<uintptr_t>(x.p) % 16 != 0)
      return fail(MLP_ERR_MISALIGNED, "pointer %s is not 16-byte aligned", x.name);
  }
  return MLP_OK;
}

mlp_status_t check_ws(const Shape& s, void* ws, size_t ws_bytes, bool recompute = false, int32_t mode = 0) {
  if (ws == nullptr) return fail(MLP_ERR_INVALID_ARG, "workspace pointer is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(MLP_ERR_MISALIGNED, "workspace is not 256-byte aligned");
  const size_t need = mode_workspace_bytes(s, mode, recompute);
  if (ws_bytes < need)
    return fail(MLP_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return MLP_OK;
}

// ---------------------------------------------------------------- device
struct DeviceInfo {
  bool probed = false;
  bool ok = false;
  int sms = 0;
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

mlp_status_t current_device(int& dev, int& sms) {
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MLP_ERR_UNSUPPORTED_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(MLP_ERR_UNSUPPORTED_DEVICE, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return fail(MLP_ERR_UNSUPPORTED_DEVICE, "cannot query device %d", dev);
    d.ok = (major == 10 && minor == 0);
    d.probed = true;
    if (!d.ok) return fail(MLP_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; this library runs on sm_100 only", dev,
                           major, minor);
  }
  if (!d.ok) return fail(MLP_ERR_UNSUPPORTED_DEVICE, "device %d is not sm_100", dev);
  sms = d.sms;
  return MLP_OK;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded tensor maps, cached per host thread.  A map holds only the base
// address, the extents, the row stride, the box and the element format and
// swizzle, so an entry whose key matches all of those is the map the driver
// would encode again; a launch-bound step (small batches) spends much of its
// host time encoding about seven maps per GEMM otherwise.
// Element formats of operands and outputs.
enum OpFmt : int { OP_BF16 = 0, OP_F16 = 1, OP_E4M3 = 2, OP_F32 = 3 };

struct MapKey {
  const void* ptr;
  int64_t rows, cols;
  uint32_t box0, box1;
  int kind;  // operand: OpFmt (128-byte swizzle); output: 16 + OpFmt
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && box0 == o.box0 && box1 == o.box1 && kind == o.kind;
  }
};
struct MapCache {
  static constexpr int N = 64;
  MapKey key[N];
  CUtensorMap map[N];
  bool used[N] = {};
  int next = 0;
  bool find(const MapKey& k, CUtensorMap* out) const {
    for (int i = 0; i < N; ++i)
      if (used[i] && key[i] == k) {
        *out = map[i];
        return true;
      }
    return false;
  }
  void put(const MapKey& k, const CUtensorMap& m) {
    key[next] = k;
    map[next] = m;
    used[next] = true;
    next = (next + 1) % N;
  }
};
thread_local MapCache g_map_cache;

// 2-D row-major operand [rows, cols] (cols contiguous), box of 128 bytes of
// columns (64 16-bit or 128 8-bit values) x box_rows rows, 128-byte swizzle,
// zero fill out of bounds.
mlp_status_t make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, uint32_t box_rows,
                      const char* name, int fmt = OP_BF16) {
  const cuuint64_t esz = fmt == OP_E4M3 ? 1 : 2;
  const uint32_t box_cols = static_cast<uint32_t>(128 / esz);
  const MapKey key{ptr, rows, cols, box_cols, box_rows, fmt};
  if (g_map_cache.find(key, map)) return MLP_OK;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(MLP_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esz};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapDataType dt = fmt == OP_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : (fmt == OP_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLP_ERR_CUDA, "cuTensorMapEncodeTiled failed for %s (CUresult %d)", name, (int)r);
  g_map_cache.put(key, *map);
  return MLP_OK;
}

// Output of a GEMM epilogue: row-major [rows, cols], stored in 32x32 boxes
// from the epilogue's swizzled staging tiles (bf16, fp16: 64-byte swizzle;
// fp32: 128-byte; e4m3: 32-byte; matching the staging layouts in gemm.cuh
// and fp8.cuh).
mlp_status_t make_out_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int fmt, const char* name) {
  const MapKey key{ptr, rows, cols, 32u, 32u, 16 + fmt};
  if (g_map_cache.find(key, map)) return MLP_OK;
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(MLP_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t esz = fmt == OP_F32 ? 4 : (fmt == OP_E4M3 ? 1 : 2);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esz};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapDataType dt = fmt == OP_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : fmt == OP_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : fmt == OP_F16  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = fmt == OP_F32 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : (fmt == OP_E4M3 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B);
  CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MLP_ERR_CUDA, "cuTensorMapEncodeTiled failed for output of %s (CUresult %d)", name, (int)r);
  g_map_cache.put(key, *map);
  return MLP_OK;
}

// Operand of the GEMM: `rows` is its M (or N) extent, `k` its K extent.
// K-major: stored [rows, k];  MN-major: stored [k, rows].  e4m3 operands are
// MN-major only, in 128 x 128 boxes (the 8-bit stages of F8LO).
mlp_status_t make_operand_map(CUtensorMap* map, const void* ptr, bool mn_major, int64_t rows, int64_t k,
                              uint32_t tile_rows, const char* name, int fmt) {
  if (fmt == OP_E4M3) return make_map(map, ptr, k, rows, 128u, name, fmt);
  if (mn_major) return make_map(map, ptr, k, rows, 64u, name, fmt);
  return make_map(map, ptr, rows, k, tile_rows, name, fmt);
}

// ---------------------------------------------------------------- launches
struct Operand {
  const void* p[2];  // part 0 and part 1 (part 1 = part 0 when not split)
  bool mn_major;
  int fmt[2] = {OP_BF16, OP_BF16};
};

struct GemmDesc {
  Operand a, b;
  int64_t M, N, K;  // K = shards * (K of one shard); each part spans all of K
  int shards;
  int parts;
  float* tail_scratch = nullptr;  // room for the fp32 pieces of split tiles
  size_t tail_bytes = 0;
};

// Tile order.  All resident tiles walk K in near lockstep, so DRAM traffic
// per wave is the union of their row and column operand blocks.  When one
// operand fits comfortably in L2 it stays resident and the other streams
// once.  Otherwise (the shard-sum GEMMs of the larger workloads) groups of 8
// row blocks are walked rows-first: a wave of 74 tiles then covers about 8
// row blocks by 9 column blocks, which fetches about 17% fewer DRAM bytes
// than 16 by 4.6.  Measured on B200, power-capped, fp16 operands: T=8192,
// h=12288, f=49152, t=8: Y 8.94-8.96 ms and dX 8.93-9.14 ms against
// 9.30-9.31 and 9.79-9.87 ms with groups of 16; T=16384, h=3072, f=12288:
// 0.97-0.99 / 1.02-1.04 against 0.99-1.02 / 1.03-1.08 ms; equal at T=4096,
// h=4096, f=16384.
int pick_group_m(int64_t M, int64_t N, int64_t K, int m_blocks) {
  const double l2_share = 48.0 * 1024 * 1024;
  const double a_bytes = double(M) * double(K) * 2.0, b_bytes = double(N) * double(K) * 2.0;
  if (a_bytes <= l2_share) return m_blocks;  // row operand stays resident; walk rows fastest
  if (b_bytes <= l2_share) return 1;         // column operand stays resident; walk columns fastest
  return m_blocks < 8 ? m_blocks : 8;
}

// One opt-in per kernel instantiation and device (the static state is per
// template instance).
template <bool A_MN, bool B_MN, int EPI, bool PAIR, int TN, int EW, bool DUAL, bool F8LO>
mlp_status_t ensure_kernel_setup(int dev, int sms, int* max_clusters) {
  using Cfg = TileCfg<PAIR, TN, EPI, EW, DUAL>;
  static std::mutex mu;
  static uint64_t done_mask = 0;
  static int clusters[64] = {};
  auto kernel = mlp_gemm_kernel<A_MN, B_MN, EPI, PAIR, TN, EW, DUAL, F8LO>;
  std::lock_guard<std::mutex> lk(mu);
  if (!(done_mask & (1ull << dev))) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
    int n = sms / Cfg::CTAS;
    if (PAIR) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(2 * n));
      cfg.blockDim = dim3(Cfg::THREADS);
      cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int q = 0;
      if (cudaOccupancyMaxActiveClusters(&q, kernel, &cfg) == cudaSuccess && q > 0 && q < n) n = q;
      cudaGetLastError();  // a failed occupancy query leaves no sticky error; keep the SM-count bound
    }
    clusters[dev] = n;
    done_mask |= 1ull << dev;
  }
  *max_clusters = clusters[dev];
  return MLP_OK;
}

struct Launch {
  int dev;
  int sms;
  cudaStream_t stream;
};

// Launches a helper kernel (column sums, split-tile reduce, peer reduce)
// with programmatic dependent launch, as the GEMMs: it may be scheduled while
// the previous kernel drains, and waits for it (griddepcontrol.wait) before
// its first global access.
template <typename... KArgs, typename... Args>
cudaError_t launch_helper(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <bool A_MN, bool B_MN, int EPI, int TN = 256, bool PAIR = kPair, int EW = 8, bool DUAL = false,
          bool F8LO = false>
mlp_status_t launch_gemm(const GemmDesc& g, GemmParams p, const Launch& L, const char* name) {
  using Cfg = TileCfg<PAIR, TN, EPI, EW, DUAL>;
  if (g.M == 0 || g.N == 0) return MLP_OK;
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  {
    // EPI_PEER stores with plain instructions and has no output tensor map;
    // with fp8_out the pair is (fp16, e4m3 residual)
    const int f0 = p.fp8_out ? OP_F16 : OP_BF16, f1 = p.fp8_out ? OP_E4M3 : OP_BF16;
    mlp_status_t st = p.out0 != nullptr ? make_out_map(&maps.out[0], p.out0, g.M, g.N, f0, name) : MLP_OK;
    if (st == MLP_OK && p.out1 != nullptr) st = make_out_map(&maps.out[1], p.out1, g.M, g.N, f1, name);
    if (st == MLP_OK && p.out_f32 != nullptr) st = make_out_map(&maps.out[2], p.out_f32, g.M, g.N, OP_F32, name);
    if (st != MLP_OK) return st;
  }
  for (int i = 0; i < 2; ++i) {
    mlp_status_t st = make_operand_map(&maps.a[i], g.a.p[i], A_MN, g.M, g.K, BM, name, g.a.fmt[i]);
    if (st != MLP_OK) return st;
    st = make_operand_map(&maps.b[i], g.b.p[i], B_MN, g.N, g.K, Cfg::SUB_ROWS, name, g.b.fmt[i]);
    if (st != MLP_OK) return st;
  }
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.shards = g.shards;
  p.parts = DUAL ? 1 : g.parts;  // DUAL: both halves of A in each stage, one pass over K
  p.kblocks_per_shard = static_cast<int>((g.K / g.shards + BK - 1) / BK);
  // F8LO: the fp16 part in BK-token stages, then the e4m3 part in 2*BK-token stages
  p.kb_per_unit = F8LO ? p.kblocks_per_shard + static_cast<int>((g.K + 2 * BK - 1) / (2 * BK))
                       : p.parts * p.kblocks_per_shard;
  p.m_blocks = static_cast<int>((g.M + Cfg::TILE_M - 1) / Cfg::TILE_M);
  p.n_blocks = static_cast<int>((g.N + Cfg::TILE_N - 1) / Cfg::TILE_N);
  p.num_tiles = p.m_blocks * p.n_blocks;
  p.budget_ns = g_budget_ns.load();
  p.debug_flags = g_debug_flags.load();

  int max_clusters = 0;
  mlp_status_t st = ensure_kernel_setup<A_MN, B_MN, EPI, PAIR, TN, EW, DUAL, F8LO>(L.dev, L.sms, &max_clusters);
  if (st != MLP_OK) return st;
  p.group_m = pick_group_m(g.M, g.N, g.K, p.m_blocks);
  // Work list.  Split pieces trade idle CTA pairs for extra traffic: a piece
  // stores its fp32 partial (TILE_M x TILE_N x 4 bytes) to scratch and a
  // reduce pass reads it back.  Costs are in K-slice units (one BK slice of a
  // tile's MMA); a whole tile runs U slices, a piece U/k plus
  // kPieceOverheadSlices for its store and read-back (all pairs storing
  // 256 KB at ~6 TB/s take ~3 us, about 9 slices at 1.5 GHz; measured on
  // B200: 4-way pieces of 16 slices made a 64-slice shard-sum GEMM slower).
  //  - EPI_STORE with fewer tiles than CTA pairs: every tile's K loop is cut
  //    into k pieces of consecutive K slices.
  //  - EPI_SHARD_SUM whose last wave is partial: each tile of that wave is
  //    cut into k pieces of shards/k consecutive shards (k divides t).
  // k minimises rounds(items) x (U/k + overhead) within the scratch capacity.
  constexpr double kPieceOverheadSlices = 12.0;
  p.full_tiles = p.num_tiles;
  p.tail_split = 1;
  p.kb_split = 1;
  const size_t piece_bytes = static_cast<size_t>(Cfg::TILE_M) * Cfg::TILE_N * sizeof(float);
  const size_t capacity = g.tail_scratch != nullptr ? g.tail_bytes / piece_bytes : 0;
  const int kb_per_unit = p.kb_per_unit;  // slices per shard
  auto rounds = [&](long long items) { return static_cast<double>((items + max_clusters - 1) / max_clusters); };
  // weight gradients: at least enough pieces to keep each accumulator within
  // kWgradMaxAdds additions (long token axes)
  const int64_t adds_per_unit = static_cast<int64_t>(kb_per_unit) * (BK / 16) * (DUAL ? 2 : 1);
  const int min_k = EPI == EPI_STORE ? static_cast<int>((adds_per_unit + kWgradMaxAdds - 1) / kWgradMaxAdds) : 1;
  if (min_k > 1 && static_cast<size_t>(min_k) * p.num_tiles > capacity)
    return fail(MLP_ERR_WORKSPACE_TOO_SMALL, "%s: %d K pieces per tile do not fit the split scratch", name, min_k);
  if (EPI == EPI_STORE && (p.num_tiles < max_clusters || min_k > 1) && capacity >= 2) {
    const double U = kb_per_unit;
    int best_k = min_k;
    double best = min_k == 1 ? U : rounds(static_cast<long long>(p.num_tiles) * min_k) * (U / min_k + kPieceOverheadSlices);
    for (int k = min_k + 1; k <= kb_per_unit / 8 && static_cast<size_t>(k) * p.num_tiles <= capacity; ++k) {
      const double cost = rounds(static_cast<long long>(p.num_tiles) * k) * (U / k + kPieceOverheadSlices);
      if (cost < best - 1e-9) {
        best = cost;
        best_k = k;
      }
    }
    if (best_k > 1) {
      p.kb_split = best_k;
      p.full_tiles = 0;
      p.tail_scratch = g.tail_scratch;
      p.scratch_elems = static_cast<long long>(g.tail_bytes / sizeof(float));
    }
  }
  if (EPI == EPI_SHARD_SUM && p.shards > 1 && capacity > 0) {
    const int tail = p.num_tiles % max_clusters;
    if (tail > 0) {
      const double U = static_cast<double>(p.shards) * kb_per_unit;
      int best_k = 1;
      double best = U;
      for (int k = 2; k <= p.shards; ++k) {
        if (p.shards % k != 0 || static_cast<size_t>(tail) * k > capacity) continue;
        const double cost = rounds(static_cast<long long>(tail) * k) * (U / k + kPieceOverheadSlices);
        if (cost < best - 1e-9) {
          best = cost;
          best_k = k;
        }
      }
      if (best_k > 1) {
        p.full_tiles = p.num_tiles - tail;
        p.tail_split = best_k;
        p.tail_scratch = g.tail_scratch;
        p.scratch_elems = static_cast<long long>(g.tail_bytes / sizeof(float));
      }
    }
  }
  p.num_work = p.kb_split > 1 ? p.num_tiles * p.kb_split
                             : p.full_tiles + (p.num_tiles - p.full_tiles) * p.tail_split;
  const int clusters = p.num_work < max_clusters ? p.num_work : max_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see grid_wait_prerequisites
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = Cfg::CTAS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * Cfg::CTAS));
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = L.stream;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, mlp_gemm_kernel<A_MN, B_MN, EPI, PAIR, TN, EW, DUAL, F8LO>, maps, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, name);
  g_launches.fetch_add(1);
  if (p.tail_split > 1 || p.kb_split > 1) {
    const int first = p.kb_split > 1 ? 0 : p.full_tiles;
    const int tiles = p.num_tiles - first;
    const int split = p.kb_split > 1 ? p.kb_split : p.tail_split;
    const long long threads = static_cast<long long>(tiles) * Cfg::TILE_M * (Cfg::TILE_N / 8);
    e = launch_helper(split_reduce_kernel<Cfg::TILE_M, Cfg::TILE_N>, dim3(static_cast<unsigned>((threads + 255) / 256)),
                      dim3(256), L.stream, p, first, tiles, split);
    if (e != cudaSuccess) return cuda_fail(e, "split_reduce");
    g_launches.fetch_add(1);
  }
  return MLP_OK;
}

// `partial_elems` is the size of the partial-sum buffer and `status` the
// workspace status word (NULL: none); both serve the bounds-checking build.
mlp_status_t launch_colsum_final(const float* partial, int chunks, int64_t C, void* out, cudaStream_t stream,
                                 size_t partial_elems, unsigned int* status) {
  cudaError_t e = launch_helper(colsum_final, dim3(static_cast<unsigned>((C + 31) / 32)), dim3(32, 8), stream, partial,
                                chunks, static_cast<int>(C), static_cast<__nv_bfloat16*>(out),
                                static_cast<long long>(partial_elems), status);
  if (e != cudaSuccess) return cuda_fail(e, "colsum_final");
  g_launches.fetch_add(1);
  return MLP_OK;
}

mlp_status_t launch_colsum(const void* m, int64_t R, int64_t C, void* out, float* partial, cudaStream_t stream,
                           size_t partial_elems, unsigned int* status) {
  if (R == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, static_cast<size_t>(C) * 2, stream);
    return e == cudaSuccess ? MLP_OK : cuda_fail(e, "cudaMemsetAsync(bias gradient)");
  }
  const int chunks = static_cast<int>(colsum_chunks(R));
  dim3 grid1(static_cast<unsigned>((C + COLSUM_COLS_PER_BLOCK - 1) / COLSUM_COLS_PER_BLOCK), chunks);
  cudaError_t e = launch_helper(colsum_partial, grid1, dim3(32, COLSUM_PHASES), stream,
                                static_cast<const __nv_bfloat16*>(m), static_cast<int>(R), static_cast<int>(C), partial,
                                static_cast<long long>(partial_elems), status);
  if (e != cudaSuccess) return cuda_fail(e, "colsum_partial");
  g_launches.fetch_add(1);
  return launch_colsum_final(partial, chunks, C, out, stream, partial_elems, status);
}

mlp_status_t zero_fill(void* p, size_t bytes, cudaStream_t s, const char* what) {
  cudaError_t e = cudaMemsetAsync(p, 0, bytes, s);
  return e == cudaSuccess ? MLP_OK : cuda_fail(e, what);
}

GemmParams base_params(void* ws) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.status = static_cast<unsigned int*>(ws);
  return p;
}

Operand one(const void* p, bool mn) { return Operand{{p, p}, mn}; }
Operand pair(const void* hi, const void* lo, bool mn) { return Operand{{hi, lo != nullptr ? lo : hi}, mn}; }
float* partials(void* ws, const Shape& s) {
  return reinterpret_cast<float*>(static_cast<char*>(ws) + partial_offset(s));
}
float* tail_scratch(void* ws, const Shape& s) {
  return reinterpret_cast<float*>(static_cast<char*>(ws) + tail_offset(s));
}

// Synchronises the stream, then reads and clears a device status word pair
// (code, site).
mlp_status_t read_status_word(unsigned int* status, cudaStream_t cs) {
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word[2] = {0u, 0u};
  e = cudaMemcpy(word, status, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (word[0] == 0u) return MLP_OK;
  const unsigned int zero[2] = {0u, 0u};
  e = cudaMemcpy(status, zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  if (word[0] == STATUS_TIMEOUT)
    return fail(MLP_ERR_TIMEOUT, "a kernel wait ran out of its budget (site 0x%x)", word[1]);
  if (word[0] == STATUS_BOUNDS)
    return fail(MLP_ERR_BOUNDS, "an index fell outside its buffer (site 0x%x; bounds-checking build)", word[1]);
  if (word[0] == STATUS_RANGE)
    return fail(MLP_ERR_RANGE, "a value outside the range of the fp16 + e4m3 mode (site 0x%x)", word[1]);
  return fail(MLP_ERR_CUDA, "device status word holds unknown code %u", word[0]);
}

// ---------------------------------------------------------------- stages
mlp_status_t fc1_forward(const Shape& s, const void* X, const void* A, const void* a, void* Z, void* H, void* H_lo,
                         void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.out_f32 = static_cast<float*>(Z);
  p.out0 = static_cast<__nv_bfloat16*>(H);
  p.out1 = static_cast<__nv_bfloat16*>(H_lo);
  p.bias = static_cast<const __nv_bfloat16*>(a);
  GemmDesc g{one(X, false), one(A, true), s.T, s.f, s.h, 1, 1};
  if (kFc1TN == 512) {
    // 512-column tiles unless their last wave leaves clearly more CTA pairs
    // idle than 256-column tiles do (full-wave fraction of the two).
    const int pairs = L.sms / TileShape::CTAS;
    const int64_t mt = (s.T + TileShape::TILE_M - 1) / TileShape::TILE_M;
    auto wave_eff = [&](int64_t tn) {
      const int64_t tiles = mt * ((s.f + tn - 1) / tn);
      const int64_t waves = (tiles + pairs - 1) / pairs;
      return static_cast<double>(tiles) / static_cast<double>(waves * pairs);
    };
    // When even the 256-column tiles fit in one wave, they win outright: twice
    // the CTA pairs, each with half the (here unhidden) epilogue.
    const int64_t tiles256 = mt * ((s.f + 255) / 256);
    if (tiles256 > pairs && wave_eff(512) + 0.05 >= wave_eff(256))
      return launch_gemm<false, true, EPI_BIAS_GELU, kFc1TN>(g, p, L, "column-parallel forward (Z, H)");
  }
  return launch_gemm<false, true, EPI_BIAS_GELU, 256>(g, p, L, "column-parallel forward (Z, H)");
}

mlp_status_t fc2_forward(const Shape& s, const void* H, const void* H_lo, const void* B, const void* b, void* Y,
                         void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(Y);
  p.bias = static_cast<const __nv_bfloat16*>(b);
  GemmDesc g{pair(H, H_lo, false), one(B, true), s.T, s.h, s.f, s.t, H_lo != nullptr ? 2 : 1,
             tail_scratch(ws, s), split_scratch_bytes(s)};
  if (H_lo != nullptr)
    return launch_gemm<false, true, EPI_SHARD_SUM, 256, kPair, 8, kDualA>(g, p, L, "row-parallel forward + shard reduce (Y)");
  return launch_gemm<false, true, EPI_SHARD_SUM>(g, p, L, "row-parallel forward + shard reduce (Y)");
}

mlp_status_t fc2_backward_data(const Shape& s, const void* dY, const void* B, const void* Z, void* dH, void* dH_lo,
                               void* da, void* ws, const Launch& L) {
  if (s.T == 0) return da != nullptr ? zero_fill(da, static_cast<size_t>(s.f) * 2, L.stream, "cudaMemsetAsync(da)")
                                     : MLP_OK;
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dH);
  p.out1 = static_cast<__nv_bfloat16*>(dH_lo);
  p.aux = static_cast<const float*>(Z);
  p.colsum = da != nullptr ? partials(ws, s) : nullptr;
  p.colsum_elems = static_cast<long long>(partial_bytes(s) / sizeof(float));
  GemmDesc g{one(dY, false), one(B, false), s.T, s.f, s.h, 1, 1};
  // 16 epilogue warps when K = h is short enough for the epilogue (loads of
  // Z, g'(Z), the dH pair, column sums) to outlast the mainloop of a tile:
  // measured on B200, 24% faster at h = 1024, 1.4% slower at h = 4096.
  mlp_status_t st =
      s.h <= kFc2BdManyWarpsMaxK
          ? launch_gemm<false, false, EPI_GELU_GRAD, kFc2BdTN, kPair, 16>(g, p, L, "row-parallel backward data (dH, da)")
          : launch_gemm<false, false, EPI_GELU_GRAD, kFc2BdTN, kPair, 8>(g, p, L, "row-parallel backward data (dH, da)");
  if (st != MLP_OK || da == nullptr) return st;
  return launch_colsum_final(partials(ws, s), static_cast<int>(gemm_row_blocks(s.T) * 4), s.f, da, L.stream,
                             partial_bytes(s) / sizeof(float), static_cast<unsigned int*>(ws));
}

mlp_status_t fc2_backward_weight(const Shape& s, const void* H, const void* H_lo, const void* dY, void* dB, void* db,
                                 void* ws, const Launch& L) {
  mlp_status_t st;
  if (s.T == 0) {
    st = zero_fill(dB, static_cast<size_t>(s.f * s.h * 2), L.stream, "cudaMemsetAsync(dB)");
  } else {
    GemmParams p = base_params(ws);
    p.out0 = static_cast<__nv_bfloat16*>(dB);
    GemmDesc g{pair(H, H_lo, true), one(dY, true), s.f, s.h, s.T, 1, 2, tail_scratch(ws, s), split_scratch_bytes(s)};
    st = launch_gemm<true, true, EPI_STORE, kWideTN, kPair, 8, kDualA>(g, p, L, "row-parallel weight gradient (dB)");
  }
  if (st != MLP_OK || db == nullptr) return st;
  return launch_colsum(dY, s.T, s.h, db, partials(ws, s), L.stream, partial_bytes(s) / sizeof(float),
                       static_cast<unsigned int*>(ws));
}

mlp_status_t fc1_backward_data(const Shape& s, const void* dH, const void* dH_lo, const void* A, void* dX, void* ws,
                               const Launch& L) {
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dX);
  GemmDesc g{pair(dH, dH_lo, false), one(A, false), s.T, s.h, s.f, s.t, dH_lo != nullptr ? 2 : 1,
             tail_scratch(ws, s), split_scratch_bytes(s)};
  if (dH_lo != nullptr)
    return launch_gemm<false, false, EPI_SHARD_SUM, 256, kPair, 8, kDualA>(
        g, p, L, "column-parallel backward data + shard reduce (dX)");
  return launch_gemm<false, false, EPI_SHARD_SUM>(g, p, L, "column-parallel backward data + shard reduce (dX)");
}

mlp_status_t fc1_backward_weight(const Shape& s, const void* X, const void* dH, const void* dH_lo, void* dA, void* ws,
                                 const Launch& L) {
  if (s.T == 0) return zero_fill(dA, static_cast<size_t>(s.h * s.f * 2), L.stream, "cudaMemsetAsync(dA)");
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dA);
  GemmDesc g{one(X, true), pair(dH, dH_lo, true), s.h, s.f, s.T, 1, 2, tail_scratch(ws, s), split_scratch_bytes(s)};
  return launch_gemm<true, true, EPI_STORE, kWideTN>(g, p, L, "column-parallel weight gradient (dA)");
}

// ---------------------------------------------------------------- fp16 + e4m3 mode
// (fp8.cuh).  The forward casts B to fp16; the backward reduces the
// statistics the scales follow from and casts X, dY (fp16 and e4m3, scaled)
// and A (fp16); the GEMMs then run on those copies.
struct Fp8Bufs {
  void* w16;
  void* x16;
  void* x8;
  void* dy16;
  void* dy8;
  unsigned int* stats;
};

Fp8Bufs fp8_bufs(void* ws, const Shape& s, bool recompute) {
  char* w = static_cast<char*>(ws);
  char* r = w + (recompute ? recompute_workspace_bytes(s) : workspace_bytes(s));
  const Fp8Layout l = fp8_layout(s);
  return Fp8Bufs{r + l.w16, r + l.x16, r + l.x8, r + l.dy16, r + l.dy8,
                 reinterpret_cast<unsigned int*>(w + FP8_STATS_OFFSET)};
}

mlp_status_t launch_cast(const CastJobs& jobs, const unsigned int* stats, void* ws, const Launch& L) {
  long long n = 0;
  for (int j = 0; j < jobs.count; ++j) n += jobs.job[j].n;
  if (n == 0) return MLP_OK;
  cudaError_t e = launch_helper(fp8_cast_kernel, dim3(static_cast<unsigned>(L.sms * 4)), dim3(256), L.stream, jobs,
                                stats, static_cast<unsigned int*>(ws));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_cast");
  g_launches.fetch_add(1);
  return MLP_OK;
}

// B -> fp16 copy (W16), for the row-parallel forward.
mlp_status_t fp8_prepare_forward(const Shape& s, const void* B, const Fp8Bufs& q, void* ws, const Launch& L) {
  CastJobs jobs;
  memset(&jobs, 0, sizeof(jobs));
  jobs.job[0] = CastJob{static_cast<const __nv_bfloat16*>(B), static_cast<__half*>(q.w16), nullptr, s.f * s.h,
                        CAST_UNSCALED};
  jobs.count = 1;
  return launch_cast(jobs, nullptr, ws, L);
}

// Statistics of X, dY and B, then X -> (X16, X8), dY -> (dY16, dY8) and
// A -> W16.
// The statistics of X, dY and B (the scales follow from them).
mlp_status_t fp8_backward_stats(const Shape& s, const void* dY, const void* X, const void* B, const Fp8Bufs& q,
                                const Launch& L) {
  mlp_status_t st = zero_fill(q.stats, STAT_WORDS * sizeof(unsigned int), L.stream, "cudaMemsetAsync(fp8 statistics)");
  if (st != MLP_OK) return st;
  const long long rows = 2LL * s.T + s.f;
  const long long want = (rows + STATS_THREADS / 32 - 1) / (STATS_THREADS / 32);
  const long long blocks = want < 4LL * L.sms ? want : 4LL * L.sms;
  cudaError_t e = launch_helper(fp8_stats_kernel, dim3(static_cast<unsigned>(blocks)), dim3(STATS_THREADS), L.stream,
                                static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(dY),
                                static_cast<const __nv_bfloat16*>(B), static_cast<int>(s.T), static_cast<int>(s.h),
                                static_cast<int>(s.f), q.stats);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_stats");
  g_launches.fetch_add(1);
  return MLP_OK;
}

// dY -> (dY16, dY8), A -> W16, X -> (X16, X8), in the order the backward
// GEMMs need them; after fp8_backward_stats.
mlp_status_t fp8_backward_casts(const Shape& s, const void* dY, const void* X, const void* A, const Fp8Bufs& q,
                                void* ws, const Launch& L) {
  CastJobs jobs;
  memset(&jobs, 0, sizeof(jobs));
  jobs.job[0] = CastJob{static_cast<const __nv_bfloat16*>(dY), static_cast<__half*>(q.dy16),
                        static_cast<uint8_t*>(q.dy8), s.T * s.h, CAST_SY};
  jobs.job[1] = CastJob{static_cast<const __nv_bfloat16*>(A), static_cast<__half*>(q.w16), nullptr, s.h * s.f,
                        CAST_UNSCALED};
  jobs.job[2] = CastJob{static_cast<const __nv_bfloat16*>(X), static_cast<__half*>(q.x16),
                        static_cast<uint8_t*>(q.x8), s.T * s.h, CAST_SX};
  jobs.count = 3;
  return launch_cast(jobs, q.stats, ws, L);
}

// Statistics, then the copies, on one stream.
mlp_status_t fp8_prepare_backward(const Shape& s, const void* dY, const void* X, const void* A, const void* B,
                                  const Fp8Bufs& q, void* ws, const Launch& L) {
  mlp_status_t st = fp8_backward_stats(s, dY, X, B, q, L);
  return st != MLP_OK ? st : fp8_backward_casts(s, dY, X, A, q, ws, L);
}

// A second stream per device and host thread for the fp8 mode's operand
// copies inside the composite calls.  The copies are HBM-bound and the GEMMs
// leave most of the HBM bandwidth and room for one more small block on each
// SM, so running them beside the GEMMs hides them.  The fork and the join are
// events: the side stream waits for everything enqueued before the fork, and
// the GEMM that reads the copies waits for the join, so stream order is kept
// for the caller (and a CUDA graph capture follows the fork and the join).
// Created on first use with the device current; never destroyed.
struct SideLane {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
thread_local SideLane g_side[64];

mlp_status_t side_lane(int dev, SideLane** out) {
  SideLane& l = g_side[dev];
  if (l.stream == nullptr) {
    cudaError_t e = cudaStreamCreateWithFlags(&l.stream, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "creating the fp8 mode's side stream");
  }
  *out = &l;
  return MLP_OK;
}

// The side stream waits for the work enqueued on L.stream so far; returns the
// launch description of the side stream.
mlp_status_t fork_side(const Launch& L, SideLane** lane, Launch* side) {
  mlp_status_t st = side_lane(L.dev, lane);
  if (st != MLP_OK) return st;
  cudaError_t e = cudaEventRecord((*lane)->fork, L.stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent((*lane)->stream, (*lane)->fork, 0);
  if (e != cudaSuccess) return cuda_fail(e, "forking the fp8 mode's side stream");
  *side = L;
  side->stream = (*lane)->stream;
  return MLP_OK;
}

mlp_status_t record_join(SideLane* lane) {
  cudaError_t e = cudaEventRecord(lane->join, lane->stream);
  return e == cudaSuccess ? MLP_OK : cuda_fail(e, "joining the fp8 mode's side stream");
}

mlp_status_t wait_join(SideLane* lane, const Launch& L) {
  cudaError_t e = cudaStreamWaitEvent(L.stream, lane->join, 0);
  return e == cudaSuccess ? MLP_OK : cuda_fail(e, "joining the fp8 mode's side stream");
}

Operand op16(const void* p, bool mn) { return Operand{{p, p}, mn, {OP_F16, OP_F16}}; }
Operand op16_8(const void* p16, const void* p8, bool mn) { return Operand{{p16, p8}, mn, {OP_F16, OP_E4M3}}; }

// Z = X·A + a (fp32), H16 = fp16(g(Z)), H8 = e4m3((g(Z) − H16)·2^7).
// Always 256-column tiles: two accumulators let the epilogue (whose fp16 +
// e4m3 split costs more arithmetic than the bf16 pair) overlap the next
// tile's mainloop.  Measured on B200 against 512-column tiles: 0.526 vs
// 0.551 ms at T=4096, h=4096, f=16384; 1.25 vs 1.39 ms at T=16384, h=3072,
// f=12288; equal at T=8192, h=1024, f=4096.
mlp_status_t fc1_forward_fp8(const Shape& s, const void* X, const void* A, const void* a, void* Z, void* H16,
                             void* H8, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.out_f32 = static_cast<float*>(Z);
  p.out0 = static_cast<__nv_bfloat16*>(H16);
  p.out1 = static_cast<__nv_bfloat16*>(H8);
  p.bias = static_cast<const __nv_bfloat16*>(a);
  p.fp8_out = 1;
  GemmDesc g{one(X, false), one(A, true), s.T, s.f, s.h, 1, 1};
  return launch_gemm<false, true, EPI_BIAS_GELU, 256>(g, p, L, "column-parallel forward (Z, H16, H8)");
}

// Y = Σ_i H16_i·B16_i + b.
mlp_status_t fc2_forward_fp8(const Shape& s, const void* H16, const void* B16, const void* b, void* Y, void* ws,
                             const Launch& L) {
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(Y);
  p.bias = static_cast<const __nv_bfloat16*>(b);
  p.f16_ops = 1;
  GemmDesc g{op16(H16, false), op16(B16, true), s.T, s.h, s.f, s.t, 1, tail_scratch(ws, s), split_scratch_bytes(s)};
  return launch_gemm<false, true, EPI_SHARD_SUM>(g, p, L, "row-parallel forward + shard reduce (Y, fp16)");
}

// dH = (dY·Bᵀ) ⊙ g'(Z) in fp32; dH16 = fp16(dH·sH), dH8 = e4m3((dH·sH − dH16)·2^7); da from the fp32 dH.
mlp_status_t fc2_backward_data_fp8(const Shape& s, const void* dY, const void* B, const void* Z, void* dH16,
                                   void* dH8, void* da, const unsigned int* stats, void* ws, const Launch& L) {
  if (s.T == 0) return da != nullptr ? zero_fill(da, static_cast<size_t>(s.f) * 2, L.stream, "cudaMemsetAsync(da)")
                                     : MLP_OK;
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dH16);
  p.out1 = static_cast<__nv_bfloat16*>(dH8);
  p.aux = static_cast<const float*>(Z);
  p.colsum = da != nullptr ? partials(ws, s) : nullptr;
  p.colsum_elems = static_cast<long long>(partial_bytes(s) / sizeof(float));
  p.fp8_out = 1;
  p.fp8_stats = stats;
  GemmDesc g{one(dY, false), one(B, false), s.T, s.f, s.h, 1, 1};
  mlp_status_t st =
      s.h <= kFc2BdManyWarpsMaxK
          ? launch_gemm<false, false, EPI_GELU_GRAD, kFc2BdTN, kPair, 16>(g, p, L, "row-parallel backward data (dH16, dH8, da)")
          : launch_gemm<false, false, EPI_GELU_GRAD, kFc2BdTN, kPair, 8>(g, p, L, "row-parallel backward data (dH16, dH8, da)");
  if (st != MLP_OK || da == nullptr) return st;
  return launch_colsum_final(partials(ws, s), static_cast<int>(gemm_row_blocks(s.T) * 4), s.f, da, L.stream,
                             partial_bytes(s) / sizeof(float), static_cast<unsigned int*>(ws));
}

// dB = (H16ᵀ·dY16 + H8ᵀ·dY8) / sY, db = Σ_rows dY.
mlp_status_t fc2_backward_weight_fp8(const Shape& s, const void* H16, const void* H8, const void* dY16,
                                     const void* dY8, const void* dY, void* dB, void* db, const unsigned int* stats,
                                     void* ws, const Launch& L) {
  mlp_status_t st;
  if (s.T == 0) {
    st = zero_fill(dB, static_cast<size_t>(s.f * s.h * 2), L.stream, "cudaMemsetAsync(dB)");
  } else {
    GemmParams p = base_params(ws);
    p.out0 = static_cast<__nv_bfloat16*>(dB);
    p.f16_ops = 1;
    p.fp8_stats = stats;
    p.out_scale = OUT_SCALE_INV_SY;
    GemmDesc g{op16_8(H16, H8, true), op16_8(dY16, dY8, true), s.f, s.h, s.T, 1, 2, tail_scratch(ws, s),
               split_scratch_bytes(s)};
    st = launch_gemm<true, true, EPI_STORE, kWideTN, kPair, 8, false, true>(
        g, p, L, "row-parallel weight gradient (dB, fp16 + e4m3)");
  }
  if (st != MLP_OK || db == nullptr) return st;
  return launch_colsum(dY, s.T, s.h, db, partials(ws, s), L.stream, partial_bytes(s) / sizeof(float),
                       static_cast<unsigned int*>(ws));
}

// dX = (Σ_i dH16_i·A16_iᵀ) / sH.
mlp_status_t fc1_backward_data_fp8(const Shape& s, const void* dH16, const void* A16, void* dX,
                                   const unsigned int* stats, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dX);
  p.f16_ops = 1;
  p.fp8_stats = stats;
  p.out_scale = OUT_SCALE_INV_SH;
  GemmDesc g{op16(dH16, false), op16(A16, false), s.T, s.h, s.f, s.t, 1, tail_scratch(ws, s), split_scratch_bytes(s)};
  return launch_gemm<false, false, EPI_SHARD_SUM>(g, p, L, "column-parallel backward data + shard reduce (dX, fp16)");
}

// dA = (X16ᵀ·dH16 + X8ᵀ·dH8) / (sX·sH).
mlp_status_t fc1_backward_weight_fp8(const Shape& s, const void* X16, const void* X8, const void* dH16,
                                     const void* dH8, void* dA, const unsigned int* stats, void* ws, const Launch& L) {
  if (s.T == 0) return zero_fill(dA, static_cast<size_t>(s.h * s.f * 2), L.stream, "cudaMemsetAsync(dA)");
  GemmParams p = base_params(ws);
  p.out0 = static_cast<__nv_bfloat16*>(dA);
  p.f16_ops = 1;
  p.fp8_stats = stats;
  p.out_scale = OUT_SCALE_INV_SX_SH;
  GemmDesc g{op16_8(X16, X8, true), op16_8(dH16, dH8, true), s.h, s.f, s.T, 1, 2, tail_scratch(ws, s),
             split_scratch_bytes(s)};
  return launch_gemm<true, true, EPI_STORE, kWideTN, kPair, 8, false, true>(
      g, p, L, "column-parallel weight gradient (dA, fp16 + e4m3)");
}

// The whole fp16 + e4m3 backward, given the saved Z, H16, H8; dH16 and dH8
// live in the dH pair's slots of the workspace.
mlp_status_t backward_fp8(const Shape& s, const void* dY, const void* X, const void* A, const void* B, const void* Z,
                          const void* H16, const void* H8, void* dX, void* dA, void* da, void* dB, void* db, void* ws,
                          bool recompute, const Launch& L) {
  const Fp8Bufs q = fp8_bufs(ws, s, recompute);
  void* dH16 = static_cast<char*>(ws) + dh_offset();
  void* dH8 = static_cast<char*>(ws) + dh_lo_offset(s);
  mlp_status_t st;
  // statistics first (every scale needs them), then the copies on the side
  // stream beside the GeLU-derivative GEMM, joined before the first GEMM that
  // reads them (dB)
  SideLane* lane = nullptr;
  Launch side;
  if ((st = fp8_backward_stats(s, dY, X, B, q, L)) != MLP_OK) return st;
  if ((st = fork_side(L, &lane, &side)) != MLP_OK) return st;
  if ((st = fp8_backward_casts(s, dY, X, A, q, ws, side)) != MLP_OK) return st;
  if ((st = record_join(lane)) != MLP_OK) return st;
  if ((st = fc2_backward_data_fp8(s, dY, B, Z, dH16, dH8, da, q.stats, ws, L)) != MLP_OK) return st;
  if ((st = wait_join(lane, L)) != MLP_OK) return st;
  if ((st = fc2_backward_weight_fp8(s, H16, H8, q.dy16, q.dy8, dY, dB, db, q.stats, ws, L)) != MLP_OK) return st;
  if ((st = fc1_backward_data_fp8(s, dH16, q.w16, dX, q.stats, ws, L)) != MLP_OK) return st;
  return fc1_backward_weight_fp8(s, q.x16, q.x8, dH16, dH8, dA, q.stats, ws, L);
}

mlp_status_t forward_fp8(const Shape& s, const void* X, const void* A, const void* a, const void* B, const void* b,
                         void* Y, void* Z, void* H16, void* H8, void* ws, bool recompute, const Launch& L) {
  const Fp8Bufs q = fp8_bufs(ws, s, recompute);
  mlp_status_t st;
  // the fp16 copy of B on the side stream beside the column-parallel GEMM
  SideLane* lane = nullptr;
  Launch side;
  if ((st = fork_side(L, &lane, &side)) != MLP_OK) return st;
  if ((st = fp8_prepare_forward(s, B, q, ws, side)) != MLP_OK) return st;
  if ((st = record_join(lane)) != MLP_OK) return st;
  if ((st = fc1_forward_fp8(s, X, A, a, Z, H16, H8, ws, L)) != MLP_OK) return st;
  if ((st = wait_join(lane, L)) != MLP_OK) return st;
  return fc2_forward_fp8(s, H16, q.w16, b, Y, ws, L);
}

// ---------------------------------------------------------------- across GPUs
// Buffers and tile blocks of the cross-GPU shard reduction (peer.cuh).
struct PeerShape {
  int64_t rows, nbl, ncb;
};

PeerShape peer_shape(int64_t T, int64_t h, int32_t world) {
  const int64_t rows = T / world;
  return PeerShape{rows, (rows + PEER_BLOCK_ROWS - 1) / PEER_BLOCK_ROWS, (h + PEER_BLOCK_COLS - 1) / PEER_BLOCK_COLS};
}
size_t peer_recv_bytes(int64_t T, int64_t h) { return align_up(static_cast<size_t>(T * h) * sizeof(float), 256); }
size_t peer_flag_bytes(const PeerShape& ps) {
  return align_up(static_cast<size_t>(2 * ps.nbl * ps.ncb) * sizeof(unsigned int), 256);
}

mlp_status_t check_peer(const mlp_tp_peer_t* peer, int64_t T, int64_t h, PeerParams& q, long long& recv_elems) {
  if (peer == nullptr) return fail(MLP_ERR_INVALID_ARG, "peer descriptor is NULL");
  const int32_t world = peer->world, rank = peer->rank;
  if (world < 1 || world > MLP_TP_MAX_WORLD)
    return fail(MLP_ERR_INVALID_ARG, "peer world %d outside 1..%d", world, MLP_TP_MAX_WORLD);
  if (rank < 0 || rank >= world) return fail(MLP_ERR_INVALID_ARG, "peer rank %d outside 0..%d", rank, world - 1);
  if (peer->reserved != 0u) return fail(MLP_ERR_INVALID_ARG, "peer descriptor's reserved field is not 0");
  if (T % world != 0)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "T=%lld tokens do not split over %d ranks", (long long)T, world);
  const PeerShape ps = peer_shape(T, h, world);
  if (world > 1 && ps.rows % PEER_BLOCK_ROWS != 0)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "T/world=%lld token rows per rank must be a multiple of %d",
                (long long)ps.rows, PEER_BLOCK_ROWS);
  memset(&q, 0, sizeof(q));
  for (int r = 0; r < world; ++r) {
    if (peer->recv[r] == nullptr && T > 0) return fail(MLP_ERR_INVALID_ARG, "peer receive buffer %d is NULL", r);
    if (reinterpret_cast<uintptr_t>(peer->recv[r]) % 16 != 0)
      return fail(MLP_ERR_MISALIGNED, "peer receive buffer %d is not 16-byte aligned", r);
    if (peer->epoch != 0u) {
      if (peer->flags[r] == nullptr) return fail(MLP_ERR_INVALID_ARG, "peer flag block %d is NULL", r);
      if (reinterpret_cast<uintptr_t>(peer->flags[r]) % 16 != 0)
        return fail(MLP_ERR_MISALIGNED, "peer flag block %d is not 16-byte aligned", r);
    }
    q.recv[r] = static_cast<float*>(peer->recv[r]);
    q.flags[r] = static_cast<unsigned int*>(peer->flags[r]);
  }
  q.rank = rank;
  q.world = world;
  q.rows = static_cast<int>(ps.rows);
  q.nbl = static_cast<int>(ps.nbl);
  q.ncb = static_cast<int>(ps.ncb);
  q.epoch = peer->epoch;
  recv_elems = static_cast<long long>(T) * h;
  return MLP_OK;
}

mlp_status_t fc2_forward_peer(const Shape& s, const void* H, const void* H_lo, const void* B, const PeerParams& q,
                              long long recv_elems, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.peer = q;
  p.peer_recv_elems = recv_elems;
  GemmDesc g{pair(H, H_lo, false), one(B, true), s.T, s.h, s.f, 1, H_lo != nullptr ? 2 : 1};
  if (H_lo != nullptr)
    return launch_gemm<false, true, EPI_PEER, 256, kPair, 8, kDualA>(g, p, L, "row-parallel forward to the owners (P)");
  return launch_gemm<false, true, EPI_PEER>(g, p, L, "row-parallel forward to the owners (P)");
}

mlp_status_t fc1_backward_data_peer(const Shape& s, const void* dH, const void* dH_lo, const void* A,
                                    const PeerParams& q, long long recv_elems, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.peer = q;
  p.peer_recv_elems = recv_elems;
  GemmDesc g{pair(dH, dH_lo, false), one(A, false), s.T, s.h, s.f, 1, dH_lo != nullptr ? 2 : 1};
  if (dH_lo != nullptr)
    return launch_gemm<false, false, EPI_PEER, 256, kPair, 8, kDualA>(g, p, L,
                                                                     "column-parallel backward data to the owners (Q)");
  return launch_gemm<false, false, EPI_PEER>(g, p, L, "column-parallel backward data to the owners (Q)");
}

// The fp16 + e4m3 mode's row-parallel GEMMs of one rank: H16·B16 (B16 from
// the workspace) and dH16·A16ᵀ / sH (A16 and the statistics from the
// workspace), fp32 partials to the owners.
mlp_status_t fc2_forward_peer_fp8(const Shape& s, const void* H16, const void* B16, const PeerParams& q,
                                  long long recv_elems, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.peer = q;
  p.peer_recv_elems = recv_elems;
  p.f16_ops = 1;
  GemmDesc g{op16(H16, false), op16(B16, true), s.T, s.h, s.f, 1, 1};
  return launch_gemm<false, true, EPI_PEER>(g, p, L, "row-parallel forward to the owners (P, fp16)");
}

mlp_status_t fc1_backward_data_peer_fp8(const Shape& s, const void* dH16, const void* A16, const unsigned int* stats,
                                        const PeerParams& q, long long recv_elems, void* ws, const Launch& L) {
  GemmParams p = base_params(ws);
  p.peer = q;
  p.peer_recv_elems = recv_elems;
  p.f16_ops = 1;
  p.fp8_stats = stats;
  p.out_scale = OUT_SCALE_INV_SH;
  GemmDesc g{op16(dH16, false), op16(A16, false), s.T, s.h, s.f, 1, 1};
  return launch_gemm<false, false, EPI_PEER>(g, p, L, "column-parallel backward data to the owners (Q, fp16)");
}

// Common preamble: shape, pointers, workspace, device.
mlp_status_t prologue(const Shape& s, std::initializer_list<Ptr> ptrs, void* ws, size_t ws_bytes, void* stream,
                      Launch& L, bool recompute = false, int32_t mode = 0) {
  mlp_status_t st = check_shape(s);
  if (st != MLP_OK) return st;
  st = check_ptrs(ptrs);
  if (st != MLP_OK) return st;
  st = check_ws(s, ws, ws_bytes, recompute, mode);
  if (st != MLP_OK) return st;
  L.stream = static_cast<cudaStream_t>(stream);
  return current_device(L.dev, L.sms);
}

mlp_status_t check_mode(int32_t mode) {
  if (mode < MLP_TP_ACCURATE || mode > MLP_TP_FP8) return fail(MLP_ERR_INVALID_ARG, "precision mode %d out of range", mode);
  return MLP_OK;
}

// The low half of the pair feeds Y (and dX) unless the mode asks for the fast form.
const void* fc2_lo(int32_t mode, const void* H_lo) { return (mode & MLP_TP_FAST_FC2_FORWARD) ? nullptr : H_lo; }
const void* fc1_bwd_lo(int32_t mode, const void* dH_lo) {
  return (mode & MLP_TP_FAST_FC1_BACKWARD_DATA) ? nullptr : dH_lo;
}

// Status word of the allocation-free entry point (defined with it below).
mlp_status_t noalloc_check(cudaStream_t cs);

}  // namespace

// ====================================================================== C-ABI
extern "C" {

size_t mlp_tp_workspace_bytes(int64_t T, int64_t h, int64_t f, int32_t t) {
  Shape s{T, h, f, t};
  std::string saved = g_last_error;
  const bool ok = check_shape(s) == MLP_OK;
  g_last_error = saved;
  return ok ? workspace_bytes(s) : 0;
}

mlp_status_t mlp_tp_fc1_forward(const void* X, const void* A, const void* a, int64_t T, int64_t h, int64_t f,
                                int32_t t, void* Z, void* H, void* H_lo, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{X, "X", false, s.T == 0}, {A, "A", false}, {a, "a", false}, {Z, "Z", false, s.T == 0},
                                 {H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc1_forward(s, X, A, a, Z, H, H_lo, ws, L);
}

mlp_status_t mlp_tp_fc2_forward(const void* H, const void* H_lo, const void* B, const void* b, int64_t T, int64_t h,
                                int64_t f, int32_t t, void* Y, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{H, "H", false, s.T == 0}, {H_lo, "H_lo", true, s.T == 0}, {B, "B", false}, {b, "b", true},
                                 {Y, "Y", false, s.T == 0}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc2_forward(s, H, H_lo, B, b, Y, ws, L);
}

mlp_status_t mlp_tp_forward(const void* X, const void* A, const void* a, const void* B, const void* b, int64_t T,
                            int64_t h, int64_t f, int32_t t, int32_t mode, void* Y, void* Z, void* H, void* H_lo,
                            void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = check_mode(mode);
  if (st != MLP_OK) return st;
  st = prologue(s, {{X, "X", false, s.T == 0}, {A, "A", false}, {a, "a", false}, {B, "B", false}, {b, "b", false},
                    {Y, "Y", false, s.T == 0}, {Z, "Z", false, s.T == 0}, {H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}},
                ws, ws_bytes, stream, L, false, mode);
  if (st != MLP_OK) return st;
  if (mode == MLP_TP_FP8) return forward_fp8(s, X, A, a, B, b, Y, Z, H, H_lo, ws, false, L);
  st = fc1_forward(s, X, A, a, Z, H, H_lo, ws, L);
  if (st != MLP_OK) return st;
  return fc2_forward(s, H, fc2_lo(mode, H_lo), B, b, Y, ws, L);
}

mlp_status_t mlp_tp_fc2_backward_data(const void* dY, const void* B, const void* Z, int64_t T, int64_t h, int64_t f,
                                      int32_t t, void* dH, void* dH_lo, void* da, void* ws, size_t ws_bytes,
                                      void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dY, "dY", false, s.T == 0}, {B, "B", false}, {Z, "Z", false, s.T == 0}, {dH, "dH", false, s.T == 0},
                                 {dH_lo, "dH_lo", false, s.T == 0}, {da, "da", true}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc2_backward_data(s, dY, B, Z, dH, dH_lo, da, ws, L);
}

mlp_status_t mlp_tp_fc2_backward_weight(const void* H, const void* H_lo, const void* dY, int64_t T, int64_t h,
                                        int64_t f, int32_t t, void* dB, void* db, void* ws, size_t ws_bytes,
                                        void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}, {dY, "dY", false, s.T == 0}, {dB, "dB", false},
                                 {db, "db", true}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc2_backward_weight(s, H, H_lo, dY, dB, db, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_data(const void* dH, const void* dH_lo, const void* A, int64_t T, int64_t h,
                                      int64_t f, int32_t t, void* dX, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dH, "dH", false, s.T == 0}, {dH_lo, "dH_lo", true, s.T == 0}, {A, "A", false}, {dX, "dX", false, s.T == 0}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc1_backward_data(s, dH, dH_lo, A, dX, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_weight(const void* X, const void* dH, const void* dH_lo, int64_t T, int64_t h,
                                        int64_t f, int32_t t, void* dA, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{X, "X", false, s.T == 0}, {dH, "dH", false, s.T == 0}, {dH_lo, "dH_lo", false, s.T == 0}, {dA, "dA", false}},
                             ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc1_backward_weight(s, X, dH, dH_lo, dA, ws, L);
}

mlp_status_t mlp_tp_backward(const void* dY, const void* X, const void* A, const void* B, const void* Z, const void* H,
                             const void* H_lo, int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode, void* dX,
                             void* dA, void* da, void* dB, void* db, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = check_mode(mode);
  if (st != MLP_OK) return st;
  st = prologue(s, {{dY, "dY", false, s.T == 0}, {X, "X", false, s.T == 0}, {A, "A", false}, {B, "B", false}, {Z, "Z", false, s.T == 0},
                    {H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}, {dX, "dX", false, s.T == 0}, {dA, "dA", false}, {da, "da", true},
                    {dB, "dB", false}, {db, "db", true}},
                ws, ws_bytes, stream, L, false, mode);
  if (st != MLP_OK) return st;
  if (mode == MLP_TP_FP8) return backward_fp8(s, dY, X, A, B, Z, H, H_lo, dX, dA, da, dB, db, ws, false, L);
  void* dH = static_cast<char*>(ws) + dh_offset();
  void* dH_lo = static_cast<char*>(ws) + dh_lo_offset(s);
  if ((st = fc2_backward_data(s, dY, B, Z, dH, dH_lo, da, ws, L)) != MLP_OK) return st;
  if ((st = fc2_backward_weight(s, H, H_lo, dY, dB, db, ws, L)) != MLP_OK) return st;
  if ((st = fc1_backward_data(s, dH, fc1_bwd_lo(mode, dH_lo), A, dX, ws, L)) != MLP_OK) return st;
  return fc1_backward_weight(s, X, dH, dH_lo, dA, ws, L);
}

size_t mlp_tp_recompute_workspace_bytes(int64_t T, int64_t h, int64_t f, int32_t t) {
  Shape s{T, h, f, t};
  std::string saved = g_last_error;
  const bool ok = check_shape(s) == MLP_OK;
  g_last_error = saved;
  return ok ? recompute_workspace_bytes(s) : 0;
}

mlp_status_t mlp_tp_forward_recompute(const void* X, const void* A, const void* a, const void* B, const void* b,
                                      int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode, void* Y, void* ws,
                                      size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = check_mode(mode);
  if (st != MLP_OK) return st;
  st = prologue(s, {{X, "X", false, s.T == 0}, {A, "A", false}, {a, "a", false}, {B, "B", false}, {b, "b", false},
                    {Y, "Y", false, s.T == 0}},
                ws, ws_bytes, stream, L, true, mode);
  if (st != MLP_OK) return st;
  char* w = static_cast<char*>(ws);
  void* Z = w + recompute_z_offset(s);
  void* H = w + recompute_h_offset(s);
  void* H_lo = w + recompute_hlo_offset(s);
  if (mode == MLP_TP_FP8) return forward_fp8(s, X, A, a, B, b, Y, Z, H, H_lo, ws, true, L);
  if ((st = fc1_forward(s, X, A, a, Z, H, H_lo, ws, L)) != MLP_OK) return st;
  return fc2_forward(s, H, fc2_lo(mode, H_lo), B, b, Y, ws, L);
}

mlp_status_t mlp_tp_backward_recompute(const void* dY, const void* X, const void* A, const void* a, const void* B,
                                       int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode, void* dX, void* dA,
                                       void* da, void* dB, void* db, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = check_mode(mode);
  if (st != MLP_OK) return st;
  st = prologue(s, {{dY, "dY", false, s.T == 0}, {X, "X", false, s.T == 0}, {A, "A", false}, {a, "a", false},
                    {B, "B", false}, {dX, "dX", false, s.T == 0}, {dA, "dA", false}, {da, "da", true},
                    {dB, "dB", false}, {db, "db", true}},
                ws, ws_bytes, stream, L, true, mode);
  if (st != MLP_OK) return st;
  char* w = static_cast<char*>(ws);
  void* Z = w + recompute_z_offset(s);
  void* H = w + recompute_h_offset(s);
  void* H_lo = w + recompute_hlo_offset(s);
  void* dH = w + dh_offset();
  void* dH_lo = w + dh_lo_offset(s);
  // recompute the activations the forward did not keep, then the backward
  if (mode == MLP_TP_FP8) {
    if ((st = fc1_forward_fp8(s, X, A, a, Z, H, H_lo, ws, L)) != MLP_OK) return st;
    return backward_fp8(s, dY, X, A, B, Z, H, H_lo, dX, dA, da, dB, db, ws, true, L);
  }
  if ((st = fc1_forward(s, X, A, a, Z, H, H_lo, ws, L)) != MLP_OK) return st;
  if ((st = fc2_backward_data(s, dY, B, Z, dH, dH_lo, da, ws, L)) != MLP_OK) return st;
  if ((st = fc2_backward_weight(s, H, H_lo, dY, dB, db, ws, L)) != MLP_OK) return st;
  if ((st = fc1_backward_data(s, dH, fc1_bwd_lo(mode, dH_lo), A, dX, ws, L)) != MLP_OK) return st;
  return fc1_backward_weight(s, X, dH, dH_lo, dA, ws, L);
}

size_t mlp_tp_workspace_bytes_mode(int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode) {
  Shape s{T, h, f, t};
  std::string saved = g_last_error;
  const bool ok = check_shape(s) == MLP_OK && check_mode(mode) == MLP_OK;
  g_last_error = saved;
  return ok ? mode_workspace_bytes(s, mode, false) : 0;
}

size_t mlp_tp_recompute_workspace_bytes_mode(int64_t T, int64_t h, int64_t f, int32_t t, int32_t mode) {
  Shape s{T, h, f, t};
  std::string saved = g_last_error;
  const bool ok = check_shape(s) == MLP_OK && check_mode(mode) == MLP_OK;
  g_last_error = saved;
  return ok ? mode_workspace_bytes(s, mode, true) : 0;
}

// ---- the fp16 + e4m3 mode, stage by stage
mlp_status_t mlp_tp_fp8_prepare_forward(const void* B, int64_t T, int64_t h, int64_t f, int32_t t, void* ws,
                                        size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{B, "B", false}}, ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fp8_prepare_forward(s, B, fp8_bufs(ws, s, false), ws, L);
}

mlp_status_t mlp_tp_fp8_prepare_backward(const void* dY, const void* X, const void* A, const void* B, int64_t T,
                                         int64_t h, int64_t f, int32_t t, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dY, "dY", false, s.T == 0}, {X, "X", false, s.T == 0}, {A, "A", false}, {B, "B", false}},
                             ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fp8_prepare_backward(s, dY, X, A, B, fp8_bufs(ws, s, false), ws, L);
}

mlp_status_t mlp_tp_fc1_forward_fp8(const void* X, const void* A, const void* a, int64_t T, int64_t h, int64_t f,
                                    int32_t t, void* Z, void* H, void* H_lo, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{X, "X", false, s.T == 0}, {A, "A", false}, {a, "a", false}, {Z, "Z", false, s.T == 0},
                                 {H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}},
                             ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fc1_forward_fp8(s, X, A, a, Z, H, H_lo, ws, L);
}

mlp_status_t mlp_tp_fc2_forward_fp8(const void* H, const void* b, int64_t T, int64_t h, int64_t f, int32_t t, void* Y,
                                    void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{H, "H", false, s.T == 0}, {b, "b", true}, {Y, "Y", false, s.T == 0}}, ws, ws_bytes,
                             stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fc2_forward_fp8(s, H, fp8_bufs(ws, s, false).w16, b, Y, ws, L);
}

mlp_status_t mlp_tp_fc2_backward_data_fp8(const void* dY, const void* B, const void* Z, int64_t T, int64_t h,
                                          int64_t f, int32_t t, void* dH, void* dH_lo, void* da, void* ws,
                                          size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dY, "dY", false, s.T == 0}, {B, "B", false}, {Z, "Z", false, s.T == 0},
                                 {dH, "dH", false, s.T == 0}, {dH_lo, "dH_lo", false, s.T == 0}, {da, "da", true}},
                             ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fc2_backward_data_fp8(s, dY, B, Z, dH, dH_lo, da, fp8_bufs(ws, s, false).stats, ws, L);
}

mlp_status_t mlp_tp_fc2_backward_weight_fp8(const void* H, const void* H_lo, const void* dY, int64_t T, int64_t h,
                                            int64_t f, int32_t t, void* dB, void* db, void* ws, size_t ws_bytes,
                                            void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{H, "H", false, s.T == 0}, {H_lo, "H_lo", false, s.T == 0}, {dY, "dY", false, s.T == 0},
                                 {dB, "dB", false}, {db, "db", true}},
                             ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  const Fp8Bufs q = fp8_bufs(ws, s, false);
  return fc2_backward_weight_fp8(s, H, H_lo, q.dy16, q.dy8, dY, dB, db, q.stats, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_data_fp8(const void* dH, int64_t T, int64_t h, int64_t f, int32_t t, void* dX,
                                          void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dH, "dH", false, s.T == 0}, {dX, "dX", false, s.T == 0}}, ws, ws_bytes, stream, L,
                             false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  const Fp8Bufs q = fp8_bufs(ws, s, false);
  return fc1_backward_data_fp8(s, dH, q.w16, dX, q.stats, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_weight_fp8(const void* dH, const void* dH_lo, int64_t T, int64_t h, int64_t f,
                                            int32_t t, void* dA, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, f, t};
  Launch L;
  mlp_status_t st = prologue(s, {{dH, "dH", false, s.T == 0}, {dH_lo, "dH_lo", false, s.T == 0}, {dA, "dA", false}},
                             ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  const Fp8Bufs q = fp8_bufs(ws, s, false);
  return fc1_backward_weight_fp8(s, q.x16, q.x8, dH, dH_lo, dA, q.stats, ws, L);
}

mlp_status_t mlp_tp_check(void* ws, void* stream) {
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (ws == nullptr) return noalloc_check(cs);
  return read_status_word(static_cast<unsigned int*>(ws), cs);
}

const char* mlp_tp_status_string(mlp_status_t status) {
  switch (status) {
    case MLP_OK: return "MLP_OK";
    case MLP_ERR_INVALID_ARG: return "MLP_ERR_INVALID_ARG";
    case MLP_ERR_UNSUPPORTED_SHAPE: return "MLP_ERR_UNSUPPORTED_SHAPE";
    case MLP_ERR_MISALIGNED: return "MLP_ERR_MISALIGNED";
    case MLP_ERR_WORKSPACE_TOO_SMALL: return "MLP_ERR_WORKSPACE_TOO_SMALL";
    case MLP_ERR_UNSUPPORTED_DEVICE: return "MLP_ERR_UNSUPPORTED_DEVICE";
    case MLP_ERR_CUDA: return "MLP_ERR_CUDA";
    case MLP_ERR_BOUNDS: return "MLP_ERR_BOUNDS";
    case MLP_ERR_TIMEOUT: return "MLP_ERR_TIMEOUT";
    case MLP_ERR_RANGE: return "MLP_ERR_RANGE";
  }
  return "MLP_ERR_UNKNOWN";
}

const char* mlp_tp_last_error(void) { return g_last_error.c_str(); }

uint64_t mlp_tp_launch_count(void) { return g_launches.load(); }

void mlp_tp_set_wait_budget_ns(uint64_t ns) { g_budget_ns.store(ns < 1000000ull ? 1000000ull : ns); }

void mlp_tp_set_debug_flags(uint32_t flags) { g_debug_flags.store(flags); }

size_t mlp_tp_peer_recv_bytes(int64_t T, int64_t h, int32_t world) {
  if (T < 0 || h < 64 || h % 64 != 0 || world < 1 || world > MLP_TP_MAX_WORLD || T % world != 0) return 0;
  return peer_recv_bytes(T, h);
}

size_t mlp_tp_peer_flag_bytes(int64_t T, int64_t h, int32_t world) {
  if (T < 0 || h < 64 || h % 64 != 0 || world < 1 || world > MLP_TP_MAX_WORLD || T % world != 0) return 0;
  return peer_flag_bytes(peer_shape(T, h, world));
}

mlp_status_t mlp_tp_fc2_forward_peer(const void* H, const void* H_lo, const void* B, int64_t T, int64_t h, int64_t fs,
                                     const mlp_tp_peer_t* peer, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, fs, 1};
  Launch L;
  PeerParams q;
  long long recv_elems = 0;
  mlp_status_t st = check_shape(s);
  if (st != MLP_OK || (st = check_peer(peer, T, h, q, recv_elems)) != MLP_OK) return st;
  st = prologue(s, {{H, "H", false, s.T == 0}, {H_lo, "H_lo", true, s.T == 0}, {B, "B", false}}, ws, ws_bytes, stream, L);
  if (st != MLP_OK) return st;
  return fc2_forward_peer(s, H, H_lo, B, q, recv_elems, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_data_peer(const void* dH, const void* dH_lo, const void* A, int64_t T, int64_t h,
                                           int64_t fs, const mlp_tp_peer_t* peer, void* ws, size_t ws_bytes,
                                           void* stream) {
  Shape s{T, h, fs, 1};
  Launch L;
  PeerParams q;
  long long recv_elems = 0;
  mlp_status_t st = check_shape(s);
  if (st != MLP_OK || (st = check_peer(peer, T, h, q, recv_elems)) != MLP_OK) return st;
  st = prologue(s, {{dH, "dH", false, s.T == 0}, {dH_lo, "dH_lo", true, s.T == 0}, {A, "A", false}}, ws, ws_bytes,
                stream, L);
  if (st != MLP_OK) return st;
  return fc1_backward_data_peer(s, dH, dH_lo, A, q, recv_elems, ws, L);
}

mlp_status_t mlp_tp_fc2_forward_peer_fp8(const void* H, int64_t T, int64_t h, int64_t fs, const mlp_tp_peer_t* peer,
                                         void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, fs, 1};
  Launch L;
  PeerParams q;
  long long recv_elems = 0;
  mlp_status_t st = check_shape(s);
  if (st != MLP_OK || (st = check_peer(peer, T, h, q, recv_elems)) != MLP_OK) return st;
  st = prologue(s, {{H, "H", false, s.T == 0}}, ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  return fc2_forward_peer_fp8(s, H, fp8_bufs(ws, s, false).w16, q, recv_elems, ws, L);
}

mlp_status_t mlp_tp_fc1_backward_data_peer_fp8(const void* dH, int64_t T, int64_t h, int64_t fs,
                                               const mlp_tp_peer_t* peer, void* ws, size_t ws_bytes, void* stream) {
  Shape s{T, h, fs, 1};
  Launch L;
  PeerParams q;
  long long recv_elems = 0;
  mlp_status_t st = check_shape(s);
  if (st != MLP_OK || (st = check_peer(peer, T, h, q, recv_elems)) != MLP_OK) return st;
  st = prologue(s, {{dH, "dH", false, s.T == 0}}, ws, ws_bytes, stream, L, false, MLP_TP_FP8);
  if (st != MLP_OK) return st;
  const Fp8Bufs b = fp8_bufs(ws, s, false);
  return fc1_backward_data_peer_fp8(s, dH, b.w16, b.stats, q, recv_elems, ws, L);
}

mlp_status_t mlp_tp_peer_reduce(const mlp_tp_peer_t* peer, const void* bias, int64_t T, int64_t h, void* out,
                                void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || h < 0) return fail(MLP_ERR_INVALID_ARG, "negative size T=%lld h=%lld", (long long)T, (long long)h);
  if (h < 64 || h % 64 != 0 || T > (int64_t(1) << 31) - 1 || h > (int64_t(1) << 31) - 1)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "h=%lld must be a positive multiple of 64 and T, h < 2^31", (long long)h);
  PeerParams q;
  long long recv_elems = 0;
  mlp_status_t st = check_peer(peer, T, h, q, recv_elems);
  if (st != MLP_OK) return st;
  if ((st = check_ptrs({{out, "out", false, q.rows == 0}, {bias, "bias", true}})) != MLP_OK) return st;
  if (ws == nullptr) return fail(MLP_ERR_INVALID_ARG, "workspace pointer is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(MLP_ERR_MISALIGNED, "workspace is not 256-byte aligned");
  if (ws_bytes < WS_HEADER_BYTES)
    return fail(MLP_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes, WS_HEADER_BYTES);
  int dev = 0, sms = 0;
  if ((st = current_device(dev, sms)) != MLP_OK) return st;
  const long long blocks = static_cast<long long>(q.nbl) * q.ncb;
  if (blocks == 0) return MLP_OK;
  cudaError_t e = launch_helper(peer_reduce_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256),
                                static_cast<cudaStream_t>(stream), q, static_cast<const __nv_bfloat16*>(bias),
                                static_cast<int>(h), static_cast<__nv_bfloat16*>(out), static_cast<unsigned int*>(ws),
                                static_cast<unsigned long long>(g_budget_ns.load()), recv_elems);
  if (e != cudaSuccess) return cuda_fail(e, "peer_reduce");
  g_launches.fetch_add(1);
  return MLP_OK;
}

// ---- mapping another process's buffers (CUDA IPC)
typedef CUresult (*GetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

mlp_status_t mlp_tp_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr)
    return fail(MLP_ERR_INVALID_ARG, "ipc export: NULL argument");
  static GetAddressRangeFn range_fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      range_fn = reinterpret_cast<GetAddressRangeFn>(f);
  });
  if (range_fn == nullptr) return fail(MLP_ERR_CUDA, "cuMemGetAddressRange is unavailable");
  CUdeviceptr base = 0;
  size_t size = 0;
  CUresult r = range_fn(&base, &size, reinterpret_cast<CUdeviceptr>(ptr));
  if (r != CUDA_SUCCESS) return fail(MLP_ERR_CUDA, "cuMemGetAddressRange failed (CUresult %d)", (int)r);
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  static_assert(sizeof(h) == MLP_TP_IPC_HANDLE_BYTES, "IPC handle size");
  memcpy(handle, &h, sizeof(h));
  *offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return MLP_OK;
}

mlp_status_t mlp_tp_ipc_import(const void* handle, uint64_t offset, void** ptr) {
  if (handle == nullptr || ptr == nullptr) return fail(MLP_ERR_INVALID_ARG, "ipc import: NULL argument");
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  *ptr = static_cast<char*>(base) + offset;
  return MLP_OK;
}

mlp_status_t mlp_tp_ipc_close(void* ptr, uint64_t offset) {
  if (ptr == nullptr) return fail(MLP_ERR_INVALID_ARG, "ipc close: NULL pointer");
  cudaError_t e = cudaIpcCloseMemHandle(static_cast<char*>(ptr) - offset);
  return e == cudaSuccess ? MLP_OK : cuda_fail(e, "cudaIpcCloseMemHandle");
}

}  // extern "C"

// ============================================================ allocation-free
// db = Σ_rows dY for callers that cannot allocate device memory and so have
// no workspace to hand over (see mlp_tp_fc2_bias_grad_noalloc in the
// header).  The fp32 partial sums live in this file-scope device array, which
// every GPU that loads the library holds until the process exits.
namespace {

constexpr size_t NOALLOC_MAX_PARTIALS = size_t(1) << 20;  // 4 MiB of fp32
constexpr int NOALLOC_MAX_DEVICES = 64;
static __device__ __align__(256) float g_noalloc_partials[NOALLOC_MAX_PARTIALS];
// The path's own status word (code, site), the counterpart of the one a
// workspace holds: the bounds-checking build records out-of-range indices
// here; mlp_tp_check(NULL, stream) reads and clears it.
static __device__ __align__(16) unsigned int g_noalloc_status[2];

// Host code may not use these arrays directly (on the host their names only
// stand for host-side placeholders); their device addresses are looked up
// once per device, with that device current.
struct NoallocScratch {
  float* partials = nullptr;
  unsigned int* status = nullptr;
};
NoallocScratch g_noalloc[NOALLOC_MAX_DEVICES];
std::mutex g_noalloc_mu;

mlp_status_t noalloc_scratch(int dev, NoallocScratch* out) {
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES)
    return fail(MLP_ERR_UNSUPPORTED_DEVICE, "device ordinal %d out of range for the static scratch", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocScratch& d = g_noalloc[dev];
  if (d.partials == nullptr) {
    void* p = nullptr;
    void* q = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_partials);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static column-sum scratch)");
    e = cudaGetSymbolAddress(&q, g_noalloc_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static status word)");
    d.status = static_cast<unsigned int*>(q);
    d.partials = static_cast<float*>(p);
  }
  *out = d;
  return MLP_OK;
}

}  // namespace

extern "C" mlp_status_t mlp_tp_fc2_bias_grad_noalloc(const void* dY, int64_t T, int64_t h, void* db, void* stream) {
  if (T < 0 || h < 0) return fail(MLP_ERR_INVALID_ARG, "negative size T=%lld h=%lld", (long long)T, (long long)h);
  if (h < 64 || h % 64 != 0 || T > (int64_t(1) << 31) - 1 || h > (int64_t(1) << 31) - 1)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE, "h=%lld must be a positive multiple of 64 and T, h < 2^31", (long long)h);
  const size_t need = colsum_chunks(T) * static_cast<size_t>(h);
  if (need > NOALLOC_MAX_PARTIALS)
    return fail(MLP_ERR_UNSUPPORTED_SHAPE,
                "T=%lld, h=%lld needs %zu fp32 partial sums; the allocation-free path holds at most %zu "
                "(ceil(T/%d)*h <= %zu); use mlp_tp_fc2_backward_weight with a workspace instead",
                (long long)T, (long long)h, need, NOALLOC_MAX_PARTIALS, COLSUM_ROWS_PER_CHUNK, NOALLOC_MAX_PARTIALS);
  mlp_status_t st = check_ptrs({{dY, "dY", false, T == 0}, {db, "db", false}});
  if (st != MLP_OK) return st;
  int dev = 0, sms = 0;
  if ((st = current_device(dev, sms)) != MLP_OK) return st;
  NoallocScratch scratch;
  if ((st = noalloc_scratch(dev, &scratch)) != MLP_OK) return st;
  // Pass 1 overwrites every partial it reads back in pass 2, so nothing left
  // in the array by an earlier call is ever used.
  return launch_colsum(dY, T, h, db, scratch.partials, static_cast<cudaStream_t>(stream), NOALLOC_MAX_PARTIALS,
                       scratch.status);
}

namespace {

// mlp_tp_check(NULL, stream): the allocation-free path's status word.
mlp_status_t noalloc_check(cudaStream_t cs) {
  int dev = 0, sms = 0;
  mlp_status_t st = current_device(dev, sms);
  if (st != MLP_OK) return st;
  NoallocScratch scratch;
  if ((st = noalloc_scratch(dev, &scratch)) != MLP_OK) return st;
  return read_status_word(scratch.status, cs);
}

}  // namespace
