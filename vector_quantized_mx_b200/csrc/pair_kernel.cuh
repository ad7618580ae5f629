// pair_kernel.cuh -- the native block-scaled FP4 GEMM on CTA pairs (tcgen05 cta_group::2).
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale", Figure 5 caption:
// the decoded weights run at native FP4 throughput.  Y = X . W^T with W and X
// MX-native (E2M1 codes with E8M0 scales per 32 or UE4M3 scales per 16).  Two CTAs of
// a cluster (ranks r = 0, 1) compute one 256 x 256 tile: weight rows
// n0 + 128 r .. + 127 and token rows m0 + 128 r .. + 127 are CTA r's halves of the two
// operands.  Rank 0's MMA warp issues M = 256 (weights) x N = 256 (tokens) x K = 64
// block-scaled MMAs over both CTAs' shared memory; each CTA's TMEM receives its own
// 128 weight rows x all 256 tokens.  Per stage of 256 input channels an SM thus loads
// 32 KB of operands (16 KB of weights, 16 KB of tokens) instead of the 48 KB of a
// one-CTA 128 x 256 tile with the same tensor work per SM.
//
// Copies: each CTA loads its own operand halves, its weight scale atoms and the token
// scale atoms of all 256 tokens into its own shared memory; rank 1's tensor copies
// complete on rank 0's `full` barrier (the cta_group::2 form of the tensor copy), so
// rank 0's MMA warp sees one barrier per stage for the pair.  It moves the scale
// atoms of both CTAs into their TMEM (tcgen05.cp, cta_group::2) in order with the
// MMAs, and commits the MMAs' completion to the `empty` and `accum` barriers of both
// CTAs (tcgen05.commit multicast).  No copy uses cluster multicast.
#pragma once

#include "gemv_kernel.cuh"

namespace mxc {

template <int FMT>
struct PairLayout {
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int A = kStageK / kB / 4;                 // scale atoms per 128 rows per stage
  static constexpr int X_OFF = 0;                            // [128 tokens][128 B], 128-byte swizzle
  static constexpr int W_OFF = 16384;                        // [128 weight rows][128 B]
  static constexpr int SFX_OFF = 32768;                      // A atoms: this CTA's tokens
  static constexpr int SFW_OFF = SFX_OFF + A * 512;          // 2 x A atoms: the pair's 256 weight rows
  static constexpr int BYTES = ((SFW_OFF + 2 * A * 512) + 1023) / 1024 * 1024;
  static constexpr int CTRL = 1024;                          // barriers and the TMEM slot
  // BF16 output staging: four [128 tokens][64 weight rows] sub-tiles of 128-byte rows
  // in the 128-byte swizzle, written out by tensor stores
  static constexpr int OUT_BYTES = 4 * 16384;
  static constexpr int STAGES_FIT = (227 * 1024 - 1024 - CTRL - OUT_BYTES) / BYTES;
  // TMEM: accumulator [0, 256) (lanes = this CTA's tokens, columns = the pair's 256
  // weight rows); per stage slot 12 A columns of scales (tokens: 4 A, weights: 8 A,
  // the two 128-row groups interleaved)
  static constexpr int SF_COLS = 12 * A;
  static constexpr int STAGES_TMEM = (512 - 256) / SF_COLS;
  static constexpr int STAGES = STAGES_FIT < STAGES_TMEM ? STAGES_FIT : STAGES_TMEM;
  static constexpr int OUT_OFF = CTRL + STAGES * BYTES;      // from the aligned base
  static constexpr int SMEM = 1024 + OUT_OFF + OUT_BYTES;
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM <= 232448, "shared memory");
};

// Instruction descriptor of a block-scaled E2M1 MMA with M = 256 (a CTA pair).
__host__ __device__ constexpr uint32_t idesc_mxf4_m256(int n, int scale_e8m0, int a_sf_id, int b_sf_id) {
  return (static_cast<uint32_t>(b_sf_id & 3) << 4) | (1u << 7) | (1u << 10) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(scale_e8m0 & 1) << 23) |
         (static_cast<uint32_t>(256 >> 4) << 24) | (static_cast<uint32_t>(a_sf_id & 3) << 29);
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// All prior tcgen05 operations of this thread arrive, when done, on the barrier at
// this shared-memory offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair_mxf4_block32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair_mxf4nvf4_block16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                             uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Tensor copy into this CTA's shared memory whose completion is counted on the
// mbarrier of the pair's rank 0 (bar: a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
// Two FP32 values rounded to nearest-even BF16 (the hardware conversion), lo in the
// low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Tensor store of a shared-memory box (bulk async group of this thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's committed bulk groups have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and are complete.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tc_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}


// Persistent: gridDim.x / 2 CTA pairs walk the 256 x 256 output tiles
// t = pair, pair + pairs, ... (tile t: weight rows 256 (t mod N/256), tokens
// 256 (t div N/256)); the copy ring runs on across tiles, and the MMAs of a tile
// start once the epilogue of the one before has read the accumulator.
template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_sfx, const __grid_constant__ CUtensorMap tmap_sfw,
                     const __grid_constant__ CUtensorMap tmap_y, const int y_tma,
                     const __grid_constant__ GemmParams<1> p) {
  using L = PairLayout<FMT>;
  constexpr int STAGES = L::STAGES;
  constexpr int A = L::A;
  constexpr uint32_t kTx = 32768 + 3 * A * 512;         // one CTA's bytes of a stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // [STAGES] rank 0: both CTAs' copies of a stage landed
  uint64_t* empty = full + STAGES;                      // [STAGES] the pair's MMAs of a stage are done
  uint64_t* accum = empty + STAGES;                     // a tile's MMAs are done
  uint64_t* acc_free = accum + 1;                       // rank 0: both CTAs' epilogue warps have read the tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_free + 1);
  uint8_t* stages = smem + L::CTRL;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int K = p.K;
  const int KS = K / kStageK;
  const int KB4 = K / L::kB / 4;
  const int n_pn = p.N / 256;                           // 256-row weight tiles
  const int n_tiles = n_pn * ((p.M + 255) / 256);
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;

  // ---- setup ----
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    mbar_init(acc_free, 2 * kDecWarps);                 // every epilogue warp of both CTAs
    fence_mbar_init();
    prefetch_tensormap(&tmap_x);
    prefetch_tensormap(&tmap_w);
    prefetch_tensormap(&tmap_sfx);
    prefetch_tensormap(&tmap_sfw);
  }
  if (warp == 1) {
    __syncwarp();                                       // tcgen05.alloc is warp-aligned
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                                   // the peer's barriers exist before any copy signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =============================== loader ===============================
    // Per stage each CTA loads its 128 tokens, its 128 weight rows, its tokens' scale
    // atoms and the scale atoms of the pair's 256 weight rows (tokens past the
    // activation's rows read as zeros); rank 0 expects both CTAs' bytes.
    const uint32_t bar0 = mapa_shared(smem_u32(full), 0);
    int it = 0;
    bool ok = true;
    for (int t = pair; t < n_tiles && ok; t += pairs) {
      const int n0p = (t % n_pn) * 256;
      const int m0 = (t / n_pn) * 256;
      const int xr = m0 + 128 * static_cast<int>(rank), wr = n0p + 128 * static_cast<int>(rank);
      const int ax = (m0 / 128 + static_cast<int>(rank)) * KB4, aw = (n0p / 128) * KB4;
      for (int i = 0; i < KS; ++i, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (it >= STAGES && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          uint8_t* st = stages + s * L::BYTES;
          const uint32_t bar = bar0 + s * 8;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kTx);
          tma_load_2d_pair(st + L::X_OFF, &tmap_x, i * 128, xr, bar);
          tma_load_2d_pair(st + L::W_OFF, &tmap_w, i * 128, wr, bar);
          tma_load_2d_pair(st + L::SFX_OFF, &tmap_sfx, 0, ax + i * A, bar);
          tma_load_2d_pair(st + L::SFW_OFF, &tmap_sfw, 0, aw + i * A, bar);
          tma_load_2d_pair(st + L::SFW_OFF + A * 512, &tmap_sfw, 0, aw + KB4 + i * A, bar);
        }
        __syncwarp();
      }
    }
    // Rank 0: every copy of the pair lands before the CTA can retire (rank 1's land on
    // rank 0's barrier, before the MMAs whose completion rank 1 waits for).
    if (rank == 0)
      for (int i = it > STAGES ? it - STAGES : 0; i < it; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
  } else if (warp == 1) {
    // ==================== MMA issuer (rank 0 issues for the pair) ====================
    // D[token][weight row]: the tokens are the MMA's A operand (M = 256: 128 per CTA),
    // the weight rows its B operand (N = 256: 128 per CTA).
    if (rank == 0) {
      bool ok = true;
      int it = 0, j = 0;
      for (int t = pair; t < n_tiles && ok; t += pairs, ++j) {
        if (j > 0) {                                    // the last tile's accumulator has been read
          ok = __all_sync(0xffffffffu, mbar_wait(acc_free, (j - 1) & 1));
          if (!ok) break;
          tc_fence_after();
        }
        for (int i = 0; i < KS && ok; ++i, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph));
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint8_t* st = stages + s * L::BYTES;
            const uint32_t x_s = smem_u32(st + L::X_OFF), w_s = smem_u32(st + L::W_OFF);
            const uint32_t sfx = tmem + 256 + s * L::SF_COLS, sfw = sfx + 4 * A;
            // scale atoms of both CTAs, each from its own shared memory into its TMEM
            const uint32_t sfx_s = smem_u32(st + L::SFX_OFF), sfw_s = smem_u32(st + L::SFW_OFF);
#pragma unroll
            for (int a = 0; a < A; ++a) tc_cp_pair_32x128b_warpx4(sfx + 4 * a, sdesc_sf_atom(sfx_s + a * 512));
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
              for (int a = 0; a < A; ++a)
                tc_cp_pair_32x128b_warpx4(sfw + 8 * a + 4 * g, sdesc_sf_atom(sfw_s + (g * A + a) * 512));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint64_t adesc = sdesc_kmajor_sw128(x_s + 32 * q);
              const uint64_t bdesc = sdesc_kmajor_sw128(w_s + 32 * q);
              const uint32_t acc = (i > 0 || q > 0) ? 1u : 0u;
              if constexpr (FMT == FMT_E4M3) {
                constexpr uint32_t idesc = idesc_mxf4_m256(256, 0, 0, 0);
                tc_mma_pair_mxf4nvf4_block16(tmem, adesc, bdesc, idesc, sfx + 4 * q, sfw + 8 * q, acc);
              } else {
                const int a = q >> 1;
                const uint32_t id = static_cast<uint32_t>(q & 1) * 2;
                const uint32_t idesc = idesc_mxf4_m256(256, 1, static_cast<int>(id), static_cast<int>(id));
                tc_mma_pair_mxf4_block32(tmem, adesc, bdesc, idesc, (sfx + 4 * a) | (id << 30),
                                         (sfw + 8 * a) | (id << 30), acc);
              }
            }
            tc_commit_pair(&empty[s]);                  // both CTAs may refill the stage
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair(accum);         // the tile's accumulators are final in both CTAs
        __syncwarp();
      }
    }
  } else {
    // ============================== epilogue ==============================
    // Warp w: TMEM lane quadrant w mod 4 -- tokens m0 + 128 rank + 32 (w mod 4) .. + 31,
    // one a thread -- and 64 accumulator columns (group (w - 2) / 4) of the pair's 256
    // weight rows: each thread stores 64 consecutive outputs of its token's row.
    const int qd = warp & 3;
    const int cg = (warp - 2) >> 2;
    float wts = p.w[0].w_tscale;
    if (p.w_tscale_dev) wts = *p.w_tscale_dev;
    const float scale = wts * (p.a_tscale ? *p.a_tscale : 1.0f);
    const int out_bf16 = p.out_bf16;
    const int64_t ldy = p.ldy;
    const bool vec = (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0 && (ldy % (out_bf16 ? 8 : 4)) == 0;
    const uint32_t acc_free0 = mapa_shared(smem_u32(acc_free), 0);
    uint8_t* const out_stage = smem + L::OUT_OFF;
    int j = 0;
    for (int t = pair; t < n_tiles; t += pairs, ++j) {
      const int n0p = (t % n_pn) * 256;
      const int64_t q0 = static_cast<int64_t>(t / n_pn) * 256 + 128 * rank + qd * 32;
      const bool ep_ok = mbar_wait(accum, j & 1);
      tc_fence_after();
      if (y_tma) {
        // BF16 rows through the staging sub-tiles and tensor stores: warp (qd, cg) writes
        // rows 32 qd .. + 31 of sub-tile cg (weight rows n0p + 64 cg .. + 63), 16-byte
        // chunk c of row r at chunk c ^ (r mod 8) -- the 128-byte swizzle of the store map.
        const bool live = q0 < p.M;                     // warp-uniform: some token of this quadrant exists
        // the warp's 64 columns into registers and the accumulator released at once
        // (no CTA-wide barrier on the way: the next tile's MMAs wait for this), then,
        // once the last tile's stores have read the staging, the BF16 staging stores
        uint32_t v[64];
        if (live) {
          __syncwarp();                                 // tcgen05.ld is warp-aligned
          const uint32_t ta = tmem + (static_cast<uint32_t>(qd * 32) << 16) + cg * 64;
          tmem_ld_32x32b_x32(ta, v);
          tmem_ld_32x32b_x32(ta + 32, v + 32);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {                                // the next tile's MMAs may start
          if (rank == 0) mbar_arrive(acc_free);
          else mbar_remote_arrive_signal(acc_free0);
        }
        if (threadIdx.x == 64) bulk_wait_group_read0();   // the last tile's stores have read the staging
        named_bar_sync(1, kDecThreads);
        if (live) {
          const int r = qd * 32 + lane;
          uint8_t* const row = out_stage + cg * 16384 + r * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k) {                 // 16-byte chunk k of the row
            uint32_t h2[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              h2[c] = bf16x2_rn(__uint_as_float(v[8 * k + 2 * c]) * scale, __uint_as_float(v[8 * k + 2 * c + 1]) * scale);
            *reinterpret_cast<uint4*>(row + ((k ^ (r & 7)) << 4)) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
          }
        }
        fence_proxy_async_smem();                       // staging writes -> the tensor stores' reads
        named_bar_sync(1, kDecThreads);                 // staging complete
        if (threadIdx.x == 64) {
          const int y0 = static_cast<int>(t / n_pn) * 256 + 128 * static_cast<int>(rank);
          if (ep_ok && y0 < p.M) {                      // rows past M are clipped by the map
            for (int g = 0; g < 4; ++g) tma_store_2d(&tmap_y, n0p + 64 * g, y0, out_stage + g * 16384);
            bulk_commit_group();
          }
        }
        continue;
      }
      if (q0 < p.M) {                                   // warp-uniform: some token of this quadrant exists
        const int64_t m = q0 + lane;
        const bool row_ok = ep_ok && m < p.M;
        const size_t base = static_cast<size_t>(m) * ldy + static_cast<size_t>(n0p);
#pragma unroll 1
        for (int c0 = cg * 64; c0 < cg * 64 + 64; c0 += 16) {
          uint32_t v[16];
          __syncwarp();                                 // tcgen05.ld is warp-aligned
          tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(qd * 32) << 16) + c0, v);
          tmem_ld_wait();
          if (!row_ok) continue;
          float f[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) f[c] = __uint_as_float(v[c]) * scale;
          if (out_bf16) {
            uint32_t h2[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
              h2[c] = static_cast<uint32_t>(f32_to_bf16_rne(f[2 * c])) |
                      (static_cast<uint32_t>(f32_to_bf16_rne(f[2 * c + 1])) << 16);
            uint16_t* yp = reinterpret_cast<uint16_t*>(p.y) + base + c0;
            if (vec) {
              reinterpret_cast<uint4*>(yp)[0] = make_uint4(h2[0], h2[1], h2[2], h2[3]);
              reinterpret_cast<uint4*>(yp)[1] = make_uint4(h2[4], h2[5], h2[6], h2[7]);
            } else {
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                yp[2 * c] = static_cast<uint16_t>(h2[c] & 0xFFFFu);
                yp[2 * c + 1] = static_cast<uint16_t>(h2[c] >> 16);
              }
            }
          } else {
            float* yp = reinterpret_cast<float*>(p.y) + base + c0;
            if (vec) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                reinterpret_cast<float4*>(yp)[c] = make_float4(f[4 * c], f[4 * c + 1], f[4 * c + 2], f[4 * c + 3]);
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c) yp[c] = f[c];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {                                  // this warp is done with the accumulator
        if (rank == 0) mbar_arrive(acc_free);
        else mbar_remote_arrive_signal(acc_free0);
      }
    }
  }

  if (threadIdx.x == 64) bulk_wait_group0();           // the output stores are done
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                                   // no copy, arrive or commit is left in flight
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace mxc
