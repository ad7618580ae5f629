// linear.cuh -- host-side launch of the linear-layer kernels: tensor maps, tile and
// split-K policy, workspace layout, template dispatch.
#pragma once

#include <atomic>
#include <cstring>

#include "decode_pass.cuh"
#include "pair_kernel.cuh"
#include "round_kernel.cuh"

namespace mxc {

// ------------------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime, so the library does
// not link libcuda directly).
// ------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Encoded tensor maps are cached per thread, keyed by everything that goes into the
// encoding (kind, base address, extents, strides, box): a decode step calls the
// same layers with the same buffers over and over, and encoding costs about a
// microsecond of host time per map.  A hit returns the identical 128-byte map.
struct MapKey {
  int kind;
  const void* base;
  int64_t a, b, c, d;
  bool operator==(const MapKey& o) const {
    return kind == o.kind && base == o.base && a == o.a && b == o.b && c == o.c && d == o.d;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCache {
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  int n = 0, next = 0;
  const CUtensorMap* find(const MapKey& k) const {
    for (int i = 0; i < n; ++i)
      if (key[i] == k) return &map[i];
    return nullptr;
  }
  void put(const MapKey& k, const CUtensorMap& m) {
    const int i = n < kMapCacheSize ? n++ : next;
    next = (i + 1) % kMapCacheSize;
    key[i] = k;
    map[i] = m;
  }
};
inline MapCache& map_cache() {
  static thread_local MapCache c;
  return c;
}
template <typename F>
inline bool cached_map(CUtensorMap* map, const MapKey& k, F encode) {
  MapCache& c = map_cache();
  if (const CUtensorMap* m = c.find(k)) {
    *map = *m;
    return true;
  }
  if (!encode(map)) return false;
  c.put(k, *map);
  return true;
}

// 2-D map over an FP4 matrix [rows, K/2 bytes] (row stride ld bytes); box = 128
// bytes (256 FP4 values) x box_rows rows, 128-byte swizzle, zero fill outside.
inline bool encode_fp4_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t ld,
                           int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof(*map));
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool make_fp4_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t ld, int box_rows) {
  return cached_map(map, MapKey{1, base, rows, K, ld, box_rows},
                    [&](CUtensorMap* m) { return encode_fp4_map(m, base, rows, K, ld, box_rows); });
}

// 3-D map over the same FP4 matrix seen as [K/256 stages][rows][128 bytes] (stage
// stride 128 bytes): one box = box_rows rows x box_stages consecutive 256-column
// stages, each stage a [box_rows][128 B] tile in the 128-byte swizzle.
inline bool encode_fp4_stage_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t ld,
                                 int box_rows, int box_stages) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof(*map));
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 256)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld), 128};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_stages)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool make_fp4_stage_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t ld,
                               int box_rows, int box_stages) {
  return cached_map(map, MapKey{2, base, rows, K, ld, (static_cast<int64_t>(box_stages) << 32) | box_rows},
                    [&](CUtensorMap* m) { return encode_fp4_stage_map(m, base, rows, K, ld, box_rows, box_stages); });
}

// 4-D map over packed weight indices [N/128][K/256][4][128][16] seen as 8-byte
// elements: dims {256 (one 2 KB K-quarter slab), 4 quarters, K/256 stages, N/128
// bands}; one box = quarter q of box_stages consecutive stages of one band.
inline bool encode_idx_map(CUtensorMap* map, const void* base, int64_t N, int64_t K, int box_stages) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof(*map));
  const cuuint64_t KS = static_cast<cuuint64_t>(K / 256);
  const cuuint64_t dims[4] = {256, 4, KS, static_cast<cuuint64_t>(N / 128)};
  const cuuint64_t strides[3] = {2048, 8192, KS * 8192};
  const cuuint32_t box[4] = {256, 1, static_cast<cuuint32_t>(box_stages), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 2-D map over an SF-layout scale buffer seen as rows of one 512-byte atom (64
// eight-byte elements): dims {64, atoms}; one box = box_atoms consecutive atoms.
inline bool encode_sf_map(CUtensorMap* map, const void* base, int64_t atoms, int box_atoms) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof(*map));
  const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(atoms)};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_atoms)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool make_sf_map(CUtensorMap* map, const void* base, int64_t atoms, int box_atoms) {
  return cached_map(map, MapKey{4, base, atoms, box_atoms, 0, 0},
                    [&](CUtensorMap* m) { return encode_sf_map(m, base, atoms, box_atoms); });
}

// 2-D map over a BF16 output [rows, ld] (cols used): box 64 x 128 rows, 128-byte
// swizzle (the layout of the GEMM's output staging).
inline bool encode_bf16_out_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof(*map));
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool make_bf16_out_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld) {
  return cached_map(map, MapKey{5, base, rows, cols, ld, 0},
                    [&](CUtensorMap* m) { return encode_bf16_out_map(m, base, rows, cols, ld); });
}

inline bool make_idx_map(CUtensorMap* map, const void* base, int64_t N, int64_t K, int box_stages) {
  return cached_map(map, MapKey{3, base, N, K, box_stages, 0},
                    [&](CUtensorMap* m) { return encode_idx_map(m, base, N, K, box_stages); });
}

// The dynamic shared-memory opt-in of a kernel, set once per device (the attribute
// belongs to the function on the device that is current when it is set).
template <typename Kern>
inline cudaError_t ensure_smem_attr(Kern kern, int bytes, uint64_t* done_mask) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess && bit) __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
  return err;
}

// ------------------------------------------------------------------------------------
// Policy
// ------------------------------------------------------------------------------------
constexpr int kDecodeMaxM = 16;   // M <= 16: split-K decode path with a 16-token tile
constexpr int kSMs = 148;

// Token tile (the MMA's N): 16 for decode, 256 for prefill (each decoded or loaded
// 128-row weight tile then feeds twice the tensor-core work), 128 in between.
inline int token_tile(int64_t M) { return M <= kDecodeMaxM ? 16 : M <= 128 ? 128 : 256; }

// Split-K factor of the decode path: the CTAs of one 128-row output tile form a
// cluster of `splits`; choose the largest factor (<= kMaxSplits) that keeps all
// CTAs in one wave, with at least one 256-channel stage per CTA.
inline void decode_splits(int64_t N, int64_t K, int* splits, int* ks_per_split) {
  const int n_tiles = static_cast<int>(N / kTileN);
  const int KS = static_cast<int>(K / kStageK);
  int s = kSMs / (n_tiles > 0 ? n_tiles : 1);
  s = s < 1 ? 1 : (s > kMaxSplits ? kMaxSplits : s);
  s = s > KS ? KS : s;
  const int per = (KS + s - 1) / s;
  *ks_per_split = per;
  *splits = (KS + per - 1) / per;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The linear layer's workspace starts with a fixed area of split-K arrival counters
// (one per 128-row output tile, at most 1024), which only the workspace split-K below
// touches and which it leaves zero: a workspace zeroed once keeps valid counters
// whichever calls (decode once, other shapes) used the rest of it.
constexpr size_t kSplitkCtrBytes = 4096;

// Split-K of the decode path through the workspace: when a tile would need more than
// two cluster ranks, or slices longer than the GEMV's 8 resident stages, its ranks run
// without a cluster (a cluster of four one-CTA-per-SM CTAs does not fit one wave) and
// reduce through the workspace: the tile's arrival counter (zero on entry, zero again
// at exit), and [tile][rank][128][16] FP32 scaled partials after the counter area.  Ranks: the
// fewest that give slices of at most 8 stages, and no fewer than the cluster split;
// only while all CTAs fit one wave (N = 4608, K = 8192: 9.8 us against 14.9 us on
// clusters of four; past one wave the pipelined kernel is faster: K = N = 8192 16.3
// against 16.7 us, N = 18432, K = 4096 15.1 against 17.1 us).
constexpr int kGemvWsMaxSplits = 16;
inline bool gemv_ws_split(int64_t N, int64_t K, int* splits, int* ks_per_split) {
  int s, per;
  decode_splits(N, K, &s, &per);
  if (s <= 2 && per <= kGemvMaxStages) return false;   // the two-rank cluster path
  const int KS = static_cast<int>(K / kStageK);
  int n = (KS + kGemvMaxStages - 1) / kGemvMaxStages;
  n = n < s ? s : n;
  per = (KS + n - 1) / n;
  n = (KS + per - 1) / per;
  if (n > kGemvWsMaxSplits || (N / kTileN) * n > kSMs || N / kTileN > static_cast<int64_t>(kSplitkCtrBytes / 4))
    return false;
  *splits = n;
  *ks_per_split = per;
  return true;
}
// Split-K of the fused kernel's 128-token tiles (17 to 128 tokens) through the
// workspace: with one CTA per 128-row output tile the grid would leave most SMs idle
// (K = N = 8192: 64 of 148), so each tile's K runs in `splits` slices on separate
// CTAs (as many as fill one wave, at most 4); each writes its scaled partial tile,
// [tile][rank][128 tokens][128] FP32 after the counter area, and the tile's last rank
// to arrive adds them in rank order.
constexpr int kMidMaxSplits = 4;
inline bool mid_split(int64_t M, int64_t N, int64_t K, int* splits, int* ks_per_split) {
  if (M <= kDecodeMaxM || M > 128) return false;
  const int n_tiles = static_cast<int>(N / kTileN);
  const int KS = static_cast<int>(K / kStageK);
  if (n_tiles <= 0 || n_tiles > static_cast<int>(kSplitkCtrBytes / 4)) return false;
  int s = kSMs / n_tiles;
  s = s > kMidMaxSplits ? kMidMaxSplits : s;
  s = s > KS ? KS : s;
  if (s < 2) return false;
  const int per = (KS + s - 1) / s;
  *splits = (KS + per - 1) / per;
  *ks_per_split = per;
  return *splits >= 2;
}
// the partial tiles' bytes (0 when the shape does not reduce through the workspace)
inline size_t splitk_part_bytes(int64_t M, int64_t N, int64_t K) {
  int s, per;
  if (M <= kDecodeMaxM)
    return gemv_ws_split(N, K, &s, &per) ? static_cast<size_t>(N / kTileN) * s * 128 * kGemvT * 4 : 0;
  return mid_split(M, N, K, &s, &per) ? static_cast<size_t>(N / kTileN) * s * 128 * 128 * 4 : 0;
}

// Decode once: the layer decodes its weight once per call into the workspace (native
// FP4 codes + SF-layout scales: MX-native operands, never a high-precision weight)
// and runs the native block-scaled GEMM on it, instead of the fused kernel in which
// every token tile decodes again the weight tiles it multiplies.  With 256-token
// tiles and N a multiple of 256 the native GEMM runs on CTA pairs, and decoding
// once wins from the first 256-token tile on (measured on B200, K = 4096, N = 9216:
// equal at 130 tokens, 28 vs 43 us at 768; K = N = 8192: 37 vs 42 us at 130);
// otherwise the one-CTA native GEMM makes it pay from 1024 tokens on.
constexpr int64_t kDecodeOnceMinM = 1024;
inline bool decode_once(int64_t M, int64_t N) { return M >= kDecodeOnceMinM || (M > 128 && N % 256 == 0); }

inline size_t decoded_codes_bytes(int64_t N, int64_t K) { return align_up(static_cast<size_t>(N * K / 2), 1024); }
inline size_t decoded_weight_bytes(int64_t N, int64_t K, int fmt) {
  return decoded_codes_bytes(N, K) + static_cast<size_t>(N * K / (fmt == FMT_E8M0 ? 32 : 16));
}

// Small M: the counters and the partial tiles when the shape reduces through the
// workspace (else the partial sums stay in cluster shared memory and no workspace is
// needed).  Decode once (above): the counter area, then room for the decoded weight
// (without it the fused kernel runs).
size_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt) {
  if (decode_once(M, N)) return kSplitkCtrBytes + decoded_weight_bytes(N, K, fmt);
  const size_t part = splitk_part_bytes(M, N, K);
  return part ? kSplitkCtrBytes + part : 0;
}

// QBlocks of 64 rows or 64 input channels: a 128 x 256 tile-stage draws on up to 8
// codebooks, more than the fused decoders' per-lane copies hold, so such weights are
// always decoded once (by the direct-lookup decode kernel) and run on the native GEMM.
inline bool small_qblock(int64_t qn, int64_t qk) { return qn < kTileN || qk < 128; }

size_t linear_workspace_bytes_for(int64_t M, int64_t N, int64_t K, int fmt, int64_t qn, int64_t qk) {
  return small_qblock(qn, qk) ? kSplitkCtrBytes + decoded_weight_bytes(N, K, fmt) + splitk_part_bytes(M, N, K)
                               : linear_workspace_bytes(M, N, K, fmt);
}

// The expert tile prefix and chunk prefix, (E + 1) int32 each.
size_t moe_workspace_bytes(int64_t /*M*/, int32_t E, int64_t /*N*/, int64_t /*K*/, int /*fmt*/) {
  return align_up(2 * static_cast<size_t>(E + 1) * sizeof(int32_t), 256);
}

// ------------------------------------------------------------------------------------
// Launch
// ------------------------------------------------------------------------------------
template <int FMT, int WSRC, int T, int NCB>
cudaError_t launch_gemm_ncb(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams<1>& p, dim3 grid,
                            cudaStream_t stream) {
  using L = StageLayout<FMT, WSRC, T, NCB>;
  auto kern = gemm_kernel<FMT, WSRC, T, NCB>;
  static uint64_t attr_set = 0;
  cudaError_t err = ensure_smem_attr(kern, L::SMEM, &attr_set);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (p.splits > 1 && p.red_part == nullptr) {   // the split CTAs of a tile are one cluster
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = static_cast<unsigned>(p.splits);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  err = cudaLaunchKernelEx(&cfg, kern, tx, tw, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// Two codebooks per stage only for VQ weights whose QBlock is 128 wide along K.
template <int FMT, int WSRC, int T>
cudaError_t launch_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams<1>& p, dim3 grid,
                        cudaStream_t stream) {
  if constexpr (WSRC != WSRC_NATIVE) {
    if (p.qk == 128) return launch_gemm_ncb<FMT, WSRC, T, 2>(tx, tw, p, grid, stream);
  }
  return launch_gemm_ncb<FMT, WSRC, T, 1>(tx, tw, p, grid, stream);
}

template <int FMT, int WSRC, int T>
cudaError_t dispatch_dense(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams<1>& p, dim3 grid,
                           cudaStream_t stream) {
  return launch_gemm<FMT, WSRC, T>(tx, tw, p, grid, stream);
}

template <int FMT, int WSRC>
cudaError_t dispatch_tile(int T, const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams<1>& p, dim3 grid,
                          cudaStream_t stream) {
  if (T == 16) return dispatch_dense<FMT, WSRC, 16>(tx, tw, p, grid, stream);
  if (T == 256) return dispatch_dense<FMT, WSRC, 256>(tx, tw, p, grid, stream);
  return dispatch_dense<FMT, WSRC, 128>(tx, tw, p, grid, stream);
}

// Decode GEMV: a cluster of `splits` CTAs per 128-row output tile, launched with
// programmatic stream serialization (the kernel waits for the previous kernel's
// results itself, after its setup and weight prefetch).
template <int FMT, int WSRC>
cudaError_t launch_gemv(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ti, const GemvParams& p,
                        dim3 grid, cudaStream_t stream) {
  using L = GemvLayout<FMT, WSRC>;
  auto kern = gemv_kernel<FMT, WSRC>;
  static uint64_t attr_set = 0;
  cudaError_t err = ensure_smem_attr(kern, L::SMEM, &attr_set);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (p.splits > 1 && p.red_part == nullptr) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = static_cast<unsigned>(p.splits);
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  err = cudaLaunchKernelEx(&cfg, kern, tx, tw, ti, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <int FMT>
cudaError_t dispatch_gemv(int wsrc, const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ti,
                          const GemvParams& p, dim3 grid, cudaStream_t stream) {
  if (wsrc == WSRC_VQ_DIRECT) return launch_gemv<FMT, WSRC_VQ_DIRECT>(tx, tw, ti, p, grid, stream);
  if (wsrc == WSRC_VQ_SVQ) return launch_gemv<FMT, WSRC_VQ_SVQ>(tx, tw, ti, p, grid, stream);
  if (wsrc == WSRC_VQ_QBS) return launch_gemv<FMT, WSRC_VQ_QBS>(tx, tw, ti, p, grid, stream);
  return launch_gemv<FMT, WSRC_NATIVE>(tx, tw, ti, p, grid, stream);
}

inline ExpertPtrs expert_ptrs(const LinearArgs& a) {
  ExpertPtrs e{};
  e.idx = a.w_idx;
  e.cb = a.w_cb;
  e.sf = a.w_sf;
  e.sidx = a.w_sidx;
  e.scb = a.w_scb;
  e.w_tscale = a.w_tscale;
  e.ds = a.w_ds;
  return e;
}

mxc_status run_decode_weight(const DecodeArgs& a, cudaStream_t stream);

// SMs of the current device (looked up once per device).
inline int device_sms() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kSMs;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = kSMs;
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Native weights, 256-token tiles, N a multiple of 256: CTA pairs (tcgen05 cta_group::2)
// of 256 weight rows x 256 tokens.
template <int FMT>
cudaError_t launch_pair(const CUtensorMap& tx, const CUtensorMap& tw, const GemmParams<1>& p, cudaStream_t stream) {
  using L = PairLayout<FMT>;
  const int64_t KB4 = p.K / L::kB / 4;
  CUtensorMap tsx, tsw;
  if (!make_sf_map(&tsx, p.a_sf, (static_cast<int64_t>(p.M) + 127) / 128 * KB4, L::A) ||
      !make_sf_map(&tsw, p.w[0].sf, static_cast<int64_t>(p.N) / 128 * KB4, L::A))
    return cudaErrorInvalidValue;
  // BF16 output with 16-byte aligned rows: staged tiles written by tensor stores
  CUtensorMap ty = tx;
  int y_tma = 0;
  if (p.out_bf16 && (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0 && p.ldy % 8 == 0) {
    if (!make_bf16_out_map(&ty, p.y, p.M, p.N, p.ldy)) return cudaErrorInvalidValue;
    y_tma = 1;
  }
  auto kern = gemm_pair_kernel<FMT>;
  static uint64_t attr_set = 0;
  cudaError_t err = ensure_smem_attr(kern, L::SMEM, &attr_set);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  const int64_t tiles = static_cast<int64_t>(p.N / 256) * ((p.M + 255) / 256);
  const int64_t pairs = std::min<int64_t>(device_sms() / 2, tiles);
  if (pairs <= 0) return cudaSuccess;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, tx, tw, tsx, tsw, ty, y_tma, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

mxc_status run_linear(const LinearArgs& a, cudaStream_t stream) {
  const bool small = a.wsrc != WSRC_NATIVE && small_qblock(a.qn, a.qk);
  const bool ws_ok = a.ws && a.ws_bytes >= kSplitkCtrBytes + decoded_weight_bytes(a.N, a.K, a.fmt) &&
                     reinterpret_cast<uintptr_t>(a.ws) % 16 == 0;
  if (small && !ws_ok) return MXC_ERR_WORKSPACE;
  if (a.wsrc != WSRC_NATIVE && (small || decode_once(a.M, a.N)) && ws_ok) {
    // decode once into the workspace, then the native GEMM on the decoded operands
    DecodeArgs d{};
    d.wsrc = a.wsrc;
    d.fmt = a.fmt;
    d.N = a.N;
    d.K = a.K;
    d.qn = a.qn;
    d.qk = a.qk;
    d.w_idx = a.w_idx;
    d.w_cb = a.w_cb;
    d.w_sf = a.w_sf;
    d.w_sidx = a.w_sidx;
    d.w_scb = a.w_scb;
    d.ds = a.w_ds;
    d.q_out = static_cast<uint8_t*>(a.ws) + kSplitkCtrBytes;
    d.ldq = a.K / 2;
    d.sf_out = d.q_out + decoded_codes_bytes(a.N, a.K);
    const mxc_status s = run_decode_weight(d, stream);
    if (s != MXC_OK) return s;
    LinearArgs b = a;
    b.wsrc = WSRC_NATIVE;
    b.w_q = d.q_out;
    b.w_ldq = d.ldq;
    b.w_sf = d.sf_out;
    b.w_tscale_dev = nullptr;                      // the weight tensor scale stays b.w_tscale
    b.ws_used = decoded_weight_bytes(a.N, a.K, a.fmt);   // the split-K partial tiles may follow it
    return run_linear(b, stream);
  }
  const int T = token_tile(a.M);
  const bool pair = a.wsrc == WSRC_NATIVE && T == 256 && a.N % 256 == 0;
  CUtensorMap tx, tw;
  if (!make_fp4_map(&tx, a.a_q, a.M, a.K, a.ldq, pair ? 128 : T)) return MXC_ERR_CUDA;
  if (a.wsrc == WSRC_NATIVE) {
    if (!make_fp4_map(&tw, a.w_q, a.N, a.K, a.w_ldq, 128)) return MXC_ERR_CUDA;
  } else {
    tw = tx;  // unused
  }
  GemmParams<1> p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.qn = static_cast<int>(a.qn);
  p.qk = static_cast<int>(a.qk);
  p.a_sf = a.a_sf;
  p.a_tscale = a.a_tscale;
  p.w_tscale_dev = a.w_tscale_dev;
  p.y = a.y;
  p.ldy = a.ldy;
  p.out_bf16 = a.out_bf16;
  p.splits = 1;
  p.ks_per_split = static_cast<int>(a.K / kStageK);
  p.w[0] = expert_ptrs(a);
  if (a.wsrc == WSRC_NATIVE) p.w[0].sf = a.w_sf;
  if (pair) {
    const cudaError_t err = a.fmt == FMT_E8M0 ? launch_pair<FMT_E8M0>(tx, tw, p, stream)
                                              : launch_pair<FMT_E4M3>(tx, tw, p, stream);
    return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
  }
  const int n_tiles = static_cast<int>(a.N / kTileN);
  const int m_tiles = static_cast<int>((a.M + T - 1) / T);
  if (T == 16) {
    int splits, per;
    decode_splits(a.N, a.K, &splits, &per);
    float* red_part = nullptr;
    unsigned int* red_ctr = nullptr;
    int ws_splits, ws_per;
    if (a.M <= kDecodeMaxM && gemv_ws_split(a.N, a.K, &ws_splits, &ws_per) && a.ws &&
        a.ws_bytes >= kSplitkCtrBytes + a.ws_used + splitk_part_bytes(a.M, a.N, a.K) &&
        reinterpret_cast<uintptr_t>(a.ws) % 16 == 0) {
      splits = ws_splits;
      per = ws_per;
      red_ctr = static_cast<unsigned int*>(a.ws);
      red_part = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + kSplitkCtrBytes + a.ws_used);
    }
    p.splits = splits;
    p.ks_per_split = per;
    // slices of up to kGemvMaxRounds rounds of 8 resident stages
    if (per <= kGemvMaxRounds * kGemvMaxStages && (splits <= kGemvMaxSplits || red_part)) {
      const int box = per < kGemvMaxStages ? per : kGemvMaxStages;   // stages per tensor copy: one round
      CUtensorMap tx3, ti = tw;
      if (!make_fp4_stage_map(&tx3, a.a_q, a.M, a.K, a.ldq, kGemvT, box)) return MXC_ERR_CUDA;
      if (a.wsrc != WSRC_NATIVE && !make_idx_map(&ti, a.w_idx, a.N, a.K, box)) return MXC_ERR_CUDA;
      GemvParams g{};
      g.M = p.M;
      g.N = p.N;
      g.K = p.K;
      g.qn = p.qn;
      g.qk = p.qk;
      g.a_sf = p.a_sf;
      g.a_tscale = p.a_tscale;
      g.w_tscale_dev = p.w_tscale_dev;
      g.y = p.y;
      g.ldy = p.ldy;
      g.out_bf16 = p.out_bf16;
      g.splits = splits;
      g.ks_per_split = per;
      g.w = p.w[0];
      g.red_part = red_part;
      g.red_ctr = red_ctr;
      const dim3 grid(n_tiles, m_tiles, splits);
      const cudaError_t err = a.fmt == FMT_E8M0 ? dispatch_gemv<FMT_E8M0>(a.wsrc, tx3, tw, ti, g, grid, stream)
                                                : dispatch_gemv<FMT_E4M3>(a.wsrc, tx3, tw, ti, g, grid, stream);
      return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
    }
  }
  if (T == 128) {
    int splits, per;
    if (mid_split(a.M, a.N, a.K, &splits, &per) && a.ws &&
        a.ws_bytes >= kSplitkCtrBytes + a.ws_used + splitk_part_bytes(a.M, a.N, a.K) &&
        reinterpret_cast<uintptr_t>(a.ws) % 16 == 0) {
      p.splits = splits;
      p.ks_per_split = per;
      p.red_ctr = static_cast<unsigned int*>(a.ws);
      p.red_part = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + kSplitkCtrBytes + a.ws_used);
    }
  }
  const dim3 grid(n_tiles, m_tiles, p.splits);
  cudaError_t err;
  if (a.fmt == FMT_E8M0) {
    if (a.wsrc == WSRC_VQ_DIRECT) err = dispatch_tile<FMT_E8M0, WSRC_VQ_DIRECT>(T, tx, tw, p, grid, stream);
    else if (a.wsrc == WSRC_VQ_SVQ) err = dispatch_tile<FMT_E8M0, WSRC_VQ_SVQ>(T, tx, tw, p, grid, stream);
    else if (a.wsrc == WSRC_VQ_QBS) err = dispatch_tile<FMT_E8M0, WSRC_VQ_QBS>(T, tx, tw, p, grid, stream);
    else err = dispatch_tile<FMT_E8M0, WSRC_NATIVE>(T, tx, tw, p, grid, stream);
  } else {
    if (a.wsrc == WSRC_VQ_DIRECT) err = dispatch_tile<FMT_E4M3, WSRC_VQ_DIRECT>(T, tx, tw, p, grid, stream);
    else if (a.wsrc == WSRC_VQ_SVQ) err = dispatch_tile<FMT_E4M3, WSRC_VQ_SVQ>(T, tx, tw, p, grid, stream);
    else if (a.wsrc == WSRC_VQ_QBS) err = dispatch_tile<FMT_E4M3, WSRC_VQ_QBS>(T, tx, tw, p, grid, stream);
    else err = dispatch_tile<FMT_E4M3, WSRC_NATIVE>(T, tx, tw, p, grid, stream);
  }
  return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
}

template <int FMT, int WSRC, bool SWI>
cudaError_t launch_round(const CUtensorMap& tx, const MoeRoundParams& p, dim3 grid, cudaStream_t stream) {
  using L = RoundLayout<FMT, WSRC>;
  auto kern = moe_round_kernel<FMT, WSRC, SWI>;
  static uint64_t attr_set = 0;
  cudaError_t err = ensure_smem_attr(kern, L::SMEM, &attr_set);
  if (err != cudaSuccess) return err;
  kern<<<grid, kRoundThreads, L::SMEM, stream>>>(tx, p);
  return cudaGetLastError();
}

template <bool SWI>
cudaError_t dispatch_round(int fmt, int wsrc, const CUtensorMap& tx, const MoeRoundParams& p, dim3 grid,
                           cudaStream_t stream) {
  if (fmt == FMT_E8M0) {
    if (wsrc == WSRC_VQ_DIRECT) return launch_round<FMT_E8M0, WSRC_VQ_DIRECT, SWI>(tx, p, grid, stream);
    if (wsrc == WSRC_VQ_SVQ) return launch_round<FMT_E8M0, WSRC_VQ_SVQ, SWI>(tx, p, grid, stream);
    return launch_round<FMT_E8M0, WSRC_VQ_QBS, SWI>(tx, p, grid, stream);
  }
  if (wsrc == WSRC_VQ_DIRECT) return launch_round<FMT_E4M3, WSRC_VQ_DIRECT, SWI>(tx, p, grid, stream);
  if (wsrc == WSRC_VQ_SVQ) return launch_round<FMT_E4M3, WSRC_VQ_SVQ, SWI>(tx, p, grid, stream);
  return launch_round<FMT_E4M3, WSRC_VQ_QBS, SWI>(tx, p, grid, stream);
}


// Grouped experts: the round kernel, persistent, one CTA per SM walking the (128-row
// weight band, unit of one expert's rows) items -- units of up to 256 rows, or with
// the fused SwiGLU (gate and up accumulators of one tile) of up to 128.
mxc_status run_moe_linear(const MoeArgs& m, cudaStream_t stream) {
  const LinearArgs& a = m.base;
  const size_t need = moe_workspace_bytes(a.M, m.E, a.N, a.K, a.fmt);
  if (!a.ws || a.ws_bytes < need) return MXC_ERR_WORKSPACE;
  int32_t* tile_prefix = reinterpret_cast<int32_t*>(a.ws);
  int32_t* chunk_prefix = tile_prefix + (m.E + 1);
  if (launch_group_prologue(m.offsets, m.E, a.M, tile_prefix, stream, chunk_prefix) != cudaSuccess)
    return MXC_ERR_CUDA;
  CUtensorMap tx;
  if (!make_fp4_map(&tx, a.a_q, a.M, a.K, a.ldq, kMoeXBox)) return MXC_ERR_CUDA;   // 32-row boxes
  static thread_local MoeRoundParams p;           // about 12 KB with the expert table
  std::memset(&p, 0, sizeof(p));
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.qn = static_cast<int>(a.qn);
  p.qk = static_cast<int>(a.qk);
  p.a_sf = a.a_sf;
  p.a_tscale = a.a_tscale;
  p.y = a.y;
  p.ldy = a.ldy;
  p.out_bf16 = a.out_bf16;
  p.E = m.E;
  p.offsets = m.offsets;
  p.tile_prefix = tile_prefix;
  p.chunk_prefix = chunk_prefix;
  for (int e = 0; e < m.E; ++e) {
    const mxc_weight& w = m.experts[e];
    p.w[e].idx = w.idx;
    p.w[e].cb = w.cb;
    p.w[e].sf = w.scales;
    p.w[e].sidx = w.sidx;
    p.w[e].scb = w.scb;
    p.w[e].w_tscale = w.w_tscale;
    p.w[e].ds = w.scale_group ? w.scale_group : 8;
  }
  const dim3 grid(static_cast<unsigned>(device_sms()), 1, 1);
  cudaError_t err;
  if (m.swiglu) {
    // each item owns 128 channels of h: gate rows and the matching up rows
    p.F = static_cast<int>(a.N / 2);
    p.h_q = m.h_q;
    p.ldh = m.ldh;
    p.h_sf = m.h_sf;
    p.h_tscale = m.h_tscale;
    err = dispatch_round<true>(a.fmt, a.wsrc, tx, p, grid, stream);
  } else {
    err = dispatch_round<false>(a.fmt, a.wsrc, tx, p, grid, stream);
  }
  return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
}

// Decode pass: one CTA per 128 rows x 8 stages; q_out is written by tensor stores
// (16-byte aligned base, ldq a multiple of 16: checked by the callers).
template <int FMT, int WSRC>
cudaError_t launch_decode_pass(const DecodeArgs& a, cudaStream_t stream) {
  using L = PassLayout<FMT, WSRC>;
  auto kern = decode_pass_kernel<FMT, WSRC>;
  static uint64_t attr_set = 0;
  cudaError_t err = ensure_smem_attr(kern, L::SMEM, &attr_set);
  if (err != cudaSuccess) return err;
  const int KS = static_cast<int>(a.K / kStageK);
  const int box = KS < kGemvMaxStages ? KS : kGemvMaxStages;   // stages per tensor copy
  CUtensorMap ti, tq;
  if (!make_idx_map(&ti, a.w_idx, a.N, a.K, box) || !make_fp4_stage_map(&tq, a.q_out, a.N, a.K, a.ldq, 128, box))
    return cudaErrorInvalidValue;
  ExpertPtrs w{};
  w.idx = a.w_idx;
  w.cb = a.w_cb;
  w.sf = a.w_sf;
  w.sidx = a.w_sidx;
  w.scb = a.w_scb;
  w.ds = a.ds;
  const dim3 grid(static_cast<unsigned>(a.N / kTileN), static_cast<unsigned>((KS + kGemvMaxStages - 1) / kGemvMaxStages));
  kern<<<grid, kPassThreads, L::SMEM, stream>>>(ti, tq, w, static_cast<int>(a.N), static_cast<int>(a.K),
                                                static_cast<int>(a.qn), static_cast<int>(a.qk), box, a.sf_out);
  return cudaGetLastError();
}

template <int FMT, int WSRC>
cudaError_t launch_decode_dump_small(const DecodeArgs& a, cudaStream_t stream) {
  ExpertPtrs w{};
  w.idx = a.w_idx;
  w.cb = a.w_cb;
  w.sf = a.w_sf;
  w.sidx = a.w_sidx;
  w.scb = a.w_scb;
  w.ds = a.ds;
  const dim3 grid(static_cast<unsigned>(a.N / kTileN), static_cast<unsigned>(a.K / kStageK));
  decode_dump_small_kernel<FMT, WSRC><<<grid, 128, 0, stream>>>(w, static_cast<int>(a.N), static_cast<int>(a.K),
                                                                static_cast<int>(a.qn), static_cast<int>(a.qk),
                                                                a.q_out, a.ldq, a.sf_out);
  return cudaGetLastError();
}

mxc_status run_decode_weight(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t err;
  if (small_qblock(a.qn, a.qk)) {
    if (a.fmt == FMT_E8M0) {
      err = a.wsrc == WSRC_VQ_SVQ   ? launch_decode_dump_small<FMT_E8M0, WSRC_VQ_SVQ>(a, stream)
            : a.wsrc == WSRC_VQ_QBS ? launch_decode_dump_small<FMT_E8M0, WSRC_VQ_QBS>(a, stream)
                                    : launch_decode_dump_small<FMT_E8M0, WSRC_VQ_DIRECT>(a, stream);
    } else {
      err = a.wsrc == WSRC_VQ_SVQ   ? launch_decode_dump_small<FMT_E4M3, WSRC_VQ_SVQ>(a, stream)
            : a.wsrc == WSRC_VQ_QBS ? launch_decode_dump_small<FMT_E4M3, WSRC_VQ_QBS>(a, stream)
                                    : launch_decode_dump_small<FMT_E4M3, WSRC_VQ_DIRECT>(a, stream);
    }
    return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
  }
  if (a.fmt == FMT_E8M0) {
    err = a.wsrc == WSRC_VQ_SVQ   ? launch_decode_pass<FMT_E8M0, WSRC_VQ_SVQ>(a, stream)
          : a.wsrc == WSRC_VQ_QBS ? launch_decode_pass<FMT_E8M0, WSRC_VQ_QBS>(a, stream)
                                  : launch_decode_pass<FMT_E8M0, WSRC_VQ_DIRECT>(a, stream);
  } else {
    err = a.wsrc == WSRC_VQ_SVQ   ? launch_decode_pass<FMT_E4M3, WSRC_VQ_SVQ>(a, stream)
          : a.wsrc == WSRC_VQ_QBS ? launch_decode_pass<FMT_E4M3, WSRC_VQ_QBS>(a, stream)
                                  : launch_decode_pass<FMT_E4M3, WSRC_VQ_DIRECT>(a, stream);
  }
  return err == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
}

}  // namespace mxc
