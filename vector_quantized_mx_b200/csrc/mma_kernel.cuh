// mma_kernel.cuh -- the MXCode W4A4 linear layer on sm_100a tensor cores.
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale" (abstract):
// MX-native W4A4 operands are reconstructed from VQ storage "without
// materializing intermediate high-precision weights".  Here every CTA owns a
// 128 (output channels) x T (tokens) tile of Y^T and runs a pipeline over K in
// stages of 256 input channels:
//
//   warp 0      loader: TMA of the token tile (FP4, 128-byte swizzle) and bulk
//               copies of its scale atoms, the stage's packed index tile (8 KB),
//               its QBlock codebook(s) (512 B each) and the weight scales (direct
//               atoms, or scale-VQ indices).  Native FP4 weights come by TMA.
//   warps 2..5  decoders: index -> 16-bit codebook entry (4 E2M1 codes) -> 16-byte
//               chunks of FP4 written straight into the swizzled K-major operand
//               tile the tensor core reads; PreScale+ scale indices -> scale
//               bytes in the tcgen05 scale-factor atom layout.  Then epilogue.
//   warp 1      one thread issues tcgen05.cp (scale atoms -> TMEM) and four
//               tcgen05.mma block-scaled FP4 MMAs (K = 64 each) per stage into a
//               128 x T FP32 accumulator in TMEM, and frees the stage with
//               tcgen05.commit.
//   epilogue    warps 2..5 read the accumulator with tcgen05.ld, apply the FP32
//               tensor scales and store FP32/BF16 rows of Y (or split-K partials,
//               reduced in a fixed order by the last CTA of the tile).
//
// The weight tile is the MMA's A operand (M = 128 rows of W), the token tile is
// the B operand (N = T tokens), so one kernel serves decode (T = 16) and
// prefill (T = 128/256) without a transpose.
#pragma once

#include "mxc_device.cuh"
#include "mxc_internal.h"

namespace mxc {

enum : int { WSRC_VQ_DIRECT = 0, WSRC_VQ_SVQ = 1, WSRC_NATIVE = 2 };
enum : int { FMT_E8M0 = 0, FMT_E4M3 = 1 };

struct ExpertPtrs {
  const uint8_t* idx;
  const uint16_t* cb;
  const uint8_t* sf;     // weight scales: SF layout (VQ direct, native)
  const uint8_t* sidx;   // PreScale+ scale indices (packed tiles)
  const uint8_t* scb;    // PreScale+ scale codebook [256][8]
  float w_tscale;
  int pad_;
};

template <int NEXP>
struct GemmParams {
  int M, N, K;               // M = activation rows
  int qn, qk;                // QBlock size (resolved, nonzero)
  const uint8_t* a_sf;       // activation scales, SF layout
  const float* a_tscale;     // device or null
  const float* w_tscale_dev; // native weights: device tensor scale or null
  void* y;
  int64_t ldy;
  int out_bf16;
  int splits, ks_per_split;  // split-K (1 = off)
  float* partials;           // [splits][M][N] FP32
  int* counters;             // one per output tile, zero on entry
  int E;                     // MoE
  const int32_t* offsets;
  const int32_t* tile_prefix;
  ExpertPtrs w[NEXP];
};

// Shared-memory layout of one pipeline stage.
template <int FMT, int WSRC, int T>
struct StageLayout {
  static constexpr bool kVQ = WSRC != WSRC_NATIVE;
  static constexpr bool kSVQ = WSRC == WSRC_VQ_SVQ;
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int kAtoms = kStageK / kB / 4;     // scale atoms per 128 rows per stage
  static constexpr int kXG = (T + 127) / 128;         // 128-row scale groups in the token tile
  static constexpr int kG = kStageK / (8 * kB);       // PreScale+ scale groups per row per stage
  static constexpr int W_OFF = 0;
  static constexpr int X_OFF = 16384;
  static constexpr int SFW_OFF = X_OFF + T * 128;
  static constexpr int SFX_OFF = SFW_OFF + kAtoms * 512;
  static constexpr int IDX_OFF = SFX_OFF + kXG * kAtoms * 512;
  static constexpr int CB_OFF = IDX_OFF + (kVQ ? 8192 : 0);
  static constexpr int SIDX_OFF = CB_OFF + (kVQ ? 1024 : 0);
  static constexpr int END = SIDX_OFF + (kSVQ ? 128 * kG : 0);
  static constexpr int BYTES = (END + 1023) / 1024 * 1024;
  static constexpr int CTRL = 4096;                   // barriers, TMEM slot, scale codebook
  static constexpr int BUDGET = 227 * 1024 - 1024 - CTRL;
  static constexpr int STAGES = (BUDGET / BYTES) > 8 ? 8 : (BUDGET / BYTES);
  static constexpr int SMEM = 1024 + CTRL + STAGES * BYTES;
  // TMEM columns: accumulator [0,T), weight scales [T,T+16), token scales after.
  static constexpr int COL_SFW = T;
  static constexpr int COL_SFX = T + 16;
  static constexpr int COLS_USED = T + 16 + 16 * kXG;
  static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
  static_assert(STAGES >= 2, "stage does not fit");
  static_assert(T % 16 == 0 && T >= 16 && T <= 256, "token tile");
};

constexpr int kThreads = 192;   // 6 warps

// ------------------------------------------------------------------------------------
// Decoders (shared with the decode-dump kernel)
// ------------------------------------------------------------------------------------
// One 128 x 256 weight tile: idx [128][64] bytes, codebook(s) of 256 uint16
// entries (two when the QBlock is 128 wide along K: chunks 0..3 use the first),
// output FP4 [128][128] bytes in the 128-byte swizzle (16-byte chunk j of row r
// stored at chunk j ^ (r % 8)).  dt = 0..127.
__device__ __forceinline__ void decode_w_tile(const uint8_t* __restrict__ idx,
                                              const uint16_t* __restrict__ cb, bool cb_split,
                                              uint8_t* __restrict__ wt, int dt) {
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int c = it * 128 + dt;
    const int r = c >> 3, j = c & 7;
    const uint2 iv = *reinterpret_cast<const uint2*>(idx + r * 64 + j * 8);
    const uint16_t* t = cb + ((cb_split && j >= 4) ? 256 : 0);
    const uint32_t w0 = t[iv.x & 0xFF] | (static_cast<uint32_t>(t[(iv.x >> 8) & 0xFF]) << 16);
    const uint32_t w1 = t[(iv.x >> 16) & 0xFF] | (static_cast<uint32_t>(t[iv.x >> 24]) << 16);
    const uint32_t w2 = t[iv.y & 0xFF] | (static_cast<uint32_t>(t[(iv.y >> 8) & 0xFF]) << 16);
    const uint32_t w3 = t[(iv.y >> 16) & 0xFF] | (static_cast<uint32_t>(t[iv.y >> 24]) << 16);
    *reinterpret_cast<uint4*>(wt + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(w0, w1, w2, w3);
  }
}

// PreScale+ (Table 4 caption: Ks = 256, ds = 8): the G scale-codebook indices of
// row dt select 8 scale bytes each, i.e. two 32-bit words of the scale-factor
// atoms (kb 8g..8g+3 -> atom 2g, kb 8g+4..8g+7 -> atom 2g+1).
template <int G>
__device__ __forceinline__ void decode_sf_tile(const uint8_t* __restrict__ sidx,
                                               const uint8_t* __restrict__ scb, uint8_t* __restrict__ sfw,
                                               int dt) {
  const int word = (dt & 31) * 4 + ((dt >> 5) & 3);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint32_t si = sidx[dt * G + g];
    const uint2 s8 = *reinterpret_cast<const uint2*>(scb + si * 8);
    reinterpret_cast<uint32_t*>(sfw + (2 * g) * 512)[word] = s8.x;
    reinterpret_cast<uint32_t*>(sfw + (2 * g + 1) * 512)[word] = s8.y;
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------------------
template <int FMT, int WSRC, int T, bool MOE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wq,
                const __grid_constant__ GemmParams<MOE ? kMaxGroups : 1> p) {
  using L = StageLayout<FMT, WSRC, T>;
  constexpr int STAGES = L::STAGES;
  constexpr int A = L::kAtoms;
  constexpr int XG = L::kXG;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* dec = full + STAGES;
  uint64_t* empty = dec + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 1);
  uint8_t* scb_smem = smem + 2048;
  uint8_t* stages = smem + L::CTRL;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = p.K / kStageK;
  const int KB4 = p.K / L::kB / 4;      // scale atoms per 128 rows over all of K

  // ---- which tile this CTA owns ----
  const int n_tile = blockIdx.x;
  int64_t m0, m_end;
  int sf_group0, ks_begin = 0, ks_end = KS, split = 0;
  const ExpertPtrs* wp = &p.w[0];
  if constexpr (MOE) {
    const int tile = blockIdx.y;
    if (tile >= p.tile_prefix[p.E]) return;          // beyond this call's tile count
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {                                // last expert whose first tile <= tile
      const int mid = (lo + hi + 1) >> 1;
      if (p.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    m0 = p.offsets[lo] + static_cast<int64_t>(tile - p.tile_prefix[lo]) * 128;
    m_end = p.offsets[lo + 1];
    sf_group0 = tile;
    wp = &p.w[lo];
  } else {
    m0 = static_cast<int64_t>(blockIdx.y) * T;
    m_end = p.M;
    sf_group0 = static_cast<int>(m0 / 128);
    split = blockIdx.z;
    ks_begin = split * p.ks_per_split;
    ks_end = min(KS, ks_begin + p.ks_per_split);
  }
  const int nks = ks_end - ks_begin;

  // ---- setup ----
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&dec[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmap_x);
    if constexpr (WSRC == WSRC_NATIVE) prefetch_tensormap(&tmap_wq);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (L::kSVQ) {
    for (int i = threadIdx.x; i < 512; i += kThreads)
      reinterpret_cast<uint32_t*>(scb_smem)[i] = __ldg(reinterpret_cast<const uint32_t*>(wp->scb) + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =============================== loader ===============================
    if (lane == 0) {
      const int qbn = static_cast<int>((static_cast<int64_t>(n_tile) * 128) / p.qn);
      const int cb_per_row = p.K / p.qk;
      const bool cb_split = p.qk == 128;
      uint32_t tx = T * 128 + XG * A * 512;
      if constexpr (WSRC == WSRC_NATIVE) tx += 16384 + A * 512;
      if constexpr (WSRC == WSRC_VQ_DIRECT) tx += 8192 + (cb_split ? 1024 : 512) + A * 512;
      if constexpr (WSRC == WSRC_VQ_SVQ) tx += 8192 + (cb_split ? 1024 : 512) + 128 * L::kG;
      int issued = 0;
      for (int i = 0; i < nks; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (i >= STAGES && !mbar_wait(&empty[s], ph ^ 1)) break;
        const int ks = ks_begin + i;
        uint8_t* st = stages + s * L::BYTES;
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(st + L::X_OFF, &tmap_x, ks * 128, static_cast<int>(m0), &full[s]);
#pragma unroll
        for (int g = 0; g < XG; ++g)
          bulk_load(st + L::SFX_OFF + g * A * 512,
                    p.a_sf + (static_cast<size_t>(sf_group0 + g) * KB4 + static_cast<size_t>(ks) * A) * 512,
                    A * 512, &full[s]);
        const size_t wsf = (static_cast<size_t>(n_tile) * KB4 + static_cast<size_t>(ks) * A) * 512;
        if constexpr (WSRC == WSRC_NATIVE) {
          tma_load_2d(st + L::W_OFF, &tmap_wq, ks * 128, n_tile * 128, &full[s]);
          bulk_load(st + L::SFW_OFF, wp->sf + wsf, A * 512, &full[s]);
        } else {
          const size_t tile_id = static_cast<size_t>(n_tile) * KS + ks;
          bulk_load(st + L::IDX_OFF, wp->idx + tile_id * 8192, 8192, &full[s]);
          const int qbk = cb_split ? 2 * ks : (ks * kStageK) / p.qk;
          bulk_load(st + L::CB_OFF, wp->cb + (static_cast<size_t>(qbn) * cb_per_row + qbk) * 256,
                    cb_split ? 1024 : 512, &full[s]);
          if constexpr (WSRC == WSRC_VQ_DIRECT) {
            bulk_load(st + L::SFW_OFF, wp->sf + wsf, A * 512, &full[s]);
          } else {
            bulk_load(st + L::SIDX_OFF, wp->sidx + tile_id * (128 * L::kG), 128 * L::kG, &full[s]);
          }
        }
        ++issued;
      }
      // Let every copy this warp started land before the CTA can retire.
      for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    if (lane == 0) {
      for (int i = 0; i < nks; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[s], ph)) break;
        if constexpr (L::kVQ) {
          if (!mbar_wait(&dec[s], ph)) break;
        }
        fence_proxy_async_smem();
        tc_fence_after();
        const uint8_t* st = stages + s * L::BYTES;
        const uint32_t sfw_s = smem_u32(st + L::SFW_OFF), sfx_s = smem_u32(st + L::SFX_OFF);
#pragma unroll
        for (int a = 0; a < A; ++a) tc_cp_32x128b_warpx4(tmem + L::COL_SFW + 4 * a, sdesc_sf_atom(sfw_s + a * 512));
#pragma unroll
        for (int g = 0; g < XG; ++g)
#pragma unroll
          for (int a = 0; a < A; ++a)
            tc_cp_32x128b_warpx4(tmem + L::COL_SFX + (XG == 2 ? 8 * a + 4 * g : 4 * a),
                                 sdesc_sf_atom(sfx_s + (g * A + a) * 512));
        const uint32_t w_s = smem_u32(st + L::W_OFF), x_s = smem_u32(st + L::X_OFF);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t adesc = sdesc_kmajor_sw128(w_s + 32 * j);
          const uint64_t bdesc = sdesc_kmajor_sw128(x_s + 32 * j);
          const uint32_t acc = (i > 0 || j > 0) ? 1u : 0u;
          if constexpr (FMT == FMT_E4M3) {
            constexpr uint32_t idesc = idesc_mxf4(T, 0, 0, 0);
            tc_mma_mxf4nvf4_block16(tmem, adesc, bdesc, idesc, tmem + L::COL_SFW + 4 * j,
                                    tmem + L::COL_SFX + (XG == 2 ? 8 * j : 4 * j), acc);
          } else {
            const int a = j >> 1;
            const uint32_t id = static_cast<uint32_t>(j & 1) * 2;
            const uint32_t idesc = idesc_mxf4(T, 1, static_cast<int>(id), static_cast<int>(id));
            tc_mma_mxf4_block32(tmem, adesc, bdesc, idesc, (tmem + L::COL_SFW + 4 * a) | (id << 30),
                                (tmem + L::COL_SFX + (XG == 2 ? 8 * a : 4 * a)) | (id << 30), acc);
          }
        }
        tc_commit(&empty[s]);
      }
      tc_commit(accum);
      mbar_wait(accum, 0);      // our own MMAs must finish before the CTA retires
    }
  } else {
    // ======================= decoders, then epilogue ======================
    const int dt = threadIdx.x - 64;
    if constexpr (L::kVQ) {
      const bool cb_split = p.qk == 128;
      for (int i = 0; i < nks; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[s], ph)) break;
        uint8_t* st = stages + s * L::BYTES;
        decode_w_tile(st + L::IDX_OFF, reinterpret_cast<const uint16_t*>(st + L::CB_OFF), cb_split,
                      st + L::W_OFF, dt);
        if constexpr (L::kSVQ) decode_sf_tile<L::kG>(st + L::SIDX_OFF, scb_smem, st + L::SFW_OFF, dt);
        fence_proxy_async_smem();
        mbar_arrive(&dec[s]);
      }
    }
    const bool ok = mbar_wait(accum, 0);
    tc_fence_after();
    const int qd = warp & 3;                         // TMEM lane quadrant this warp may read
    const int row = qd * 32 + lane;
    const int64_t n = static_cast<int64_t>(n_tile) * 128 + row;
    float wts = wp->w_tscale;
    if constexpr (WSRC == WSRC_NATIVE) {
      if (p.w_tscale_dev) wts = *p.w_tscale_dev;
    }
    const float scale = wts * (p.a_tscale ? *p.a_tscale : 1.0f);
    const bool partial = p.splits > 1;
#pragma unroll 1
    for (int c0 = 0; c0 < T; c0 += 16) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(qd * 32) << 16) + c0, v);
      tmem_ld_wait();
      if (!ok) continue;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int64_t m = m0 + c0 + c;
        if (m >= m_end) break;
        const float acc = __uint_as_float(v[c]);
        if (partial) {
          p.partials[(static_cast<size_t>(split) * p.M + m) * p.N + n] = acc;
        } else if (p.out_bf16) {
          reinterpret_cast<uint16_t*>(p.y)[m * p.ldy + n] = f32_to_bf16_rne(acc * scale);
        } else {
          reinterpret_cast<float*>(p.y)[m * p.ldy + n] = acc * scale;
        }
      }
    }
    if (partial && ok) {
      // Split-K: the last CTA of this output tile sums the partials in split order.
      __threadfence();
      named_bar_sync(1, 128);
      if (dt == 0) {
        const int tile_id = blockIdx.y * gridDim.x + blockIdx.x;
        *last_flag = atomicAdd(&p.counters[tile_id], 1) == p.splits - 1;
      }
      named_bar_sync(1, 128);
      if (*last_flag) {
        __threadfence();
        for (int c = 0; c < T; ++c) {
          const int64_t m = m0 + c;
          if (m >= m_end) break;
          float sum = 0.0f;
          for (int s2 = 0; s2 < p.splits; ++s2)
            sum += __ldcg(&p.partials[(static_cast<size_t>(s2) * p.M + m) * p.N + n]);
          if (p.out_bf16) {
            reinterpret_cast<uint16_t*>(p.y)[m * p.ldy + n] = f32_to_bf16_rne(sum * scale);
          } else {
            reinterpret_cast<float*>(p.y)[m * p.ldy + n] = sum * scale;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------
// Decode dump: the decoders of gemm_kernel, with the stage written back to global
// memory in plain layouts (FP4 matrix, SF layout).  Grid (N/128, K/256), 160 threads.
// ------------------------------------------------------------------------------------
template <int FMT, int WSRC>
__global__ void __launch_bounds__(160)
    decode_dump_kernel(const ExpertPtrs w, int N, int K, int qn, int qk, uint8_t* __restrict__ q_out,
                       int64_t ldq, uint8_t* __restrict__ sf_out) {
  using L = StageLayout<FMT, WSRC, 16>;
  constexpr int A = L::kAtoms;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  uint8_t* scb_smem = smem + 2048;
  uint8_t* st = smem + L::CTRL;
  const int n_tile = blockIdx.x, ks = blockIdx.y;
  const int KS = K / kStageK, KB4 = K / L::kB / 4;
  const bool cb_split = qk == 128;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if constexpr (L::kSVQ) {
    for (int i = threadIdx.x; i < 512; i += 160)
      reinterpret_cast<uint32_t*>(scb_smem)[i] = __ldg(reinterpret_cast<const uint32_t*>(w.scb) + i);
  }
  __syncthreads();
  const size_t tile_id = static_cast<size_t>(n_tile) * KS + ks;
  const size_t wsf = (static_cast<size_t>(n_tile) * KB4 + static_cast<size_t>(ks) * A) * 512;
  if (threadIdx.x == 0) {
    const uint32_t tx = 8192 + (cb_split ? 1024 : 512) + (L::kSVQ ? 128 * L::kG : A * 512);
    mbar_arrive_expect_tx(bar, tx);
    bulk_load(st + L::IDX_OFF, w.idx + tile_id * 8192, 8192, bar);
    const int qbn = static_cast<int>((static_cast<int64_t>(n_tile) * 128) / qn);
    const int qbk = cb_split ? 2 * ks : (ks * kStageK) / qk;
    bulk_load(st + L::CB_OFF, w.cb + (static_cast<size_t>(qbn) * (K / qk) + qbk) * 256, cb_split ? 1024 : 512,
              bar);
    if constexpr (L::kSVQ) {
      bulk_load(st + L::SIDX_OFF, w.sidx + tile_id * (128 * L::kG), 128 * L::kG, bar);
    } else {
      bulk_load(st + L::SFW_OFF, w.sf + wsf, A * 512, bar);
    }
  }
  const bool ok = mbar_wait(bar, 0);
  if (threadIdx.x >= 32 && ok) {
    const int dt = threadIdx.x - 32;
    decode_w_tile(st + L::IDX_OFF, reinterpret_cast<const uint16_t*>(st + L::CB_OFF), cb_split, st + L::W_OFF, dt);
    if constexpr (L::kSVQ) decode_sf_tile<L::kG>(st + L::SIDX_OFF, scb_smem, st + L::SFW_OFF, dt);
  }
  __syncthreads();
  if (threadIdx.x >= 32 && ok) {
    const int dt = threadIdx.x - 32;
    for (int it = 0; it < 8; ++it) {
      const int c = it * 128 + dt;
      const int r = c >> 3, j = c & 7;
      const uint4 v = *reinterpret_cast<const uint4*>(st + L::W_OFF + r * 128 + ((j ^ (r & 7)) << 4));
      *reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(n_tile) * 128 + r) * ldq + ks * 128 + j * 16) = v;
    }
    for (int i = dt; i < A * 32; i += 128)
      reinterpret_cast<uint4*>(sf_out + wsf)[i] = reinterpret_cast<const uint4*>(st + L::SFW_OFF)[i];
  }
}

}  // namespace mxc
