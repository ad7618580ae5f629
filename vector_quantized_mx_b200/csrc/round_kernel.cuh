// round_kernel.cuh -- the grouped-expert (MoE) MXCode W4A4 linear layer.
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale", Table 4 caption:
// the VQ-coded tensors are MoE expert weights.  A CTA owns one expert's 128-row weight
// band and a chunk of up to 256 of that expert's tokens (two 128-token tiles), and
// walks K in rounds of four 256-channel stages:
//
//   * the loader brings in each round's weight data in two parts: its codebooks,
//     scale indices and the index quarters 0-1 of its four stages, then quarters 2-3
//     and its direct scale atoms; the next round's first part is requested as soon as
//     the decoders are done with quarter 1 of this one, the second part once they are
//     done with quarter 3 (the band of every later round was prefetched into L2 at the
//     start);
//   * the decoders lay out the 32 per-lane codebook copies once per round (decoder
//     lane l decodes stage l mod 4, so lane l's copy holds that stage's codebook:
//     conflict-free lookups, as in the decode GEMV) and decode the four stages K-quarter
//     by K-quarter straight into the swizzled FP4 operand tiles; PreScale+ weight
//     scale atoms they build once per round in shared memory from the scale indices
//     and the scale codebook (the MMA warp moves them to TMEM with tcgen05.cp), the
//     PostScale-QB ones they write to TMEM themselves from the QBlock's byte;
//   * the MMA warp runs the first token tile's block-scaled MMAs (M = 128 weight rows,
//     N = 128 tokens, K = 64) quarter by quarter behind the decode, then the second
//     tile's on the same decoded weights: each weight tile is decoded once per 256
//     tokens of its expert instead of once per 128;
//   * the token operands of one tile and round (four stages, only the 32-row boxes
//     that hold the expert's rows) and its scale atoms stream through one buffer,
//     reloaded for the next tile once the MMAs that read it are done -- by a warp of
//     their own, so that the weight loader never waits for a token buffer before
//     requesting the next round's weight data.
//
// Two TMEM accumulators hold the chunk's two tiles across all rounds; the epilogue
// scales them and writes FP32 or BF16 rows of Y.  Within a tile the K order of the
// accumulation is round by round, and within a round quarter by quarter, stage by
// stage.
#pragma once

#include "gemv_kernel.cuh"

namespace mxc {

constexpr int kRoundStages = 4;       // 256-channel stages decoded together
constexpr int kChunkTiles = 2;        // 128-token tiles per work item
constexpr int kRoundEpiWarps = 4;     // epilogue warps, one per TMEM lane quadrant
constexpr int kRoundTokWarp = 2 + kDecWarps + kRoundEpiWarps;   // the token-tile loader
constexpr int kRoundThreads = 32 * (kRoundTokWarp + 1);

struct MoeRoundParams {
  int M, N, K;
  int qn, qk;                         // QBlock (resolved; qn a multiple of 128, qk >= 128)
  const uint8_t* a_sf;                // activation scales, grouped SF layout
  const float* a_tscale;              // device or null
  void* y;
  int64_t ldy;
  int out_bf16;
  int E;
  const int32_t* offsets;
  const int32_t* tile_prefix;         // [E+1] 128-row tiles before each expert
  const int32_t* chunk_prefix;        // [E+1] 256-row chunks before each expert
  // fused SwiGLU (gate/up weights [2F, K]): h = SiLU(g) u, quantized for the down
  // projection into h_q [M, ldh] and the grouped SF layout h_sf
  int F;
  uint8_t* h_q;
  int64_t ldh;
  uint8_t* h_sf;
  const float* h_tscale;              // E4M3-B16: the given FP32 tensor scale of h
  ExpertPtrs w[kMaxGroups];
};

// The expert data of a work item, copied once per item from the kernel parameters
// into shared memory (by the loader, ahead of the item): a parameter read indexed by
// the expert costs a constant-cache round trip of the order of a thousand SM clocks,
// which the loader would otherwise pay before every round's copies and the decoders
// before their first use of the scale-VQ geometry.
struct ItemSlot {
  ExpertPtrs w;
  int qbn[2];                         // codebook row of the item's band (fused SwiGLU: and of its up band)
};

template <int FMT, int WSRC>
struct RoundLayout {
  static constexpr bool kSVQ = WSRC == WSRC_VQ_SVQ;
  static constexpr bool kQBS = WSRC == WSRC_VQ_QBS;
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int A = kStageK / kB / 4;                 // scale atoms per 128 rows per stage
  static constexpr int RS = kRoundStages;
  static constexpr int W_OFF = 0;                            // RS x [128][128 B], 128-byte swizzle
  static constexpr int X_OFF = W_OFF + RS * 16384;           // RS x [128 tokens][128 B]
  static constexpr int IDX_OFF = X_OFF + RS * 16384;         // RS x 8 KB index tiles
  static constexpr int LUT_OFF = IDX_OFF + RS * 8192;        // 32 per-lane copies x 256 words
  static constexpr int CB_OFF = LUT_OFF + kGemvLutBytes;      // the round's codebooks (<= 2 per stage)
  // Weight scale data: the direct scale atoms of two rounds (by round parity); or
  // the expert's scale codebook [256][ds] (<= 8 KB), the round's scale indices
  // (<= 1 KB) and the round's scale atoms built from them (SFS_OFF, for tcgen05.cp).
  static constexpr int AUX_OFF = CB_OFF + 2 * RS * 512;
  static constexpr int SIDX_OFF = AUX_OFF + 8192;
  static constexpr int SFS_OFF = AUX_OFF + 10240;
  static constexpr int AUX_BYTES = kSVQ ? 10240 + RS * A * 512 : 16384;
  static constexpr int SFX_OFF = AUX_OFF + AUX_BYTES;        // token scale atoms of one (round, tile)
  static constexpr int TAB_OFF = SFX_OFF + RS * A * 512;     // tile and chunk prefixes, 2 (E+1) int32
  static constexpr int CTRL_OFF = TAB_OFF + 2 * (kMaxGroups + 1) * 4 + 8;
  static constexpr int EXP_OFF = CTRL_OFF + 128;             // two ItemSlots, by item parity
  static constexpr int SMEM = 1024 + CTRL_OFF + 256;
  // TMEM: accumulators of the item's two tiles [0, 256), then two buffers each of
  // weight scales (by round parity) and token scales (by (round, tile) parity), so
  // that a scale write never hits columns that MMAs still to finish read
  static constexpr int SF_COLS = RS * A * 4;
  static constexpr int COL_SFW = 2 * 128;
  static constexpr int COL_SFX = COL_SFW + 2 * SF_COLS;
  static constexpr int TMEM_COLS = 512;
  static_assert(COL_SFX + 2 * SF_COLS <= TMEM_COLS, "tensor memory");
  static_assert(2 * RS * A * 512 <= AUX_BYTES, "direct scale staging");
  static_assert(SFS_OFF % 1024 == 0, "scale atom staging");
  static_assert(CTRL_OFF % 8 == 0 && 128 + 2 * sizeof(ItemSlot) <= 256, "control area");
  static_assert(SMEM <= 232448, "shared memory");
};

// One work item: 128 weight rows (band n_tile) of expert e against one unit of its
// rows: a chunk of up to two 128-token tiles, or (fused SwiGLU, whose gate and up
// accumulators take the TMEM of two tiles) one tile.
struct RoundItem {
  int e, n_tile, nt, tile0;           // tile0: SF group of the first tile
  int64_t m0, m_end;                  // rows [m0, min(m0 + 128 nt, m_end))
};

// Item k of the launch: unit k / n_bands, band k mod n_bands (consecutive CTAs take
// the bands of one unit, which then share its token tiles in L2).  The tables are the
// shared-memory copies of the tile and chunk prefixes; UT = tiles per unit (1 or 2).
template <int UT>
__device__ __forceinline__ RoundItem round_item(int k, int n_bands, int E, const int32_t* t_tile,
                                                const int32_t* t_chunk, const int32_t* offsets, bool rows) {
  const int32_t* t_unit = UT == 1 ? t_tile : t_chunk;
  RoundItem it;
  const int unit = k / n_bands;
  it.n_tile = k - unit * n_bands;
  int lo = 0, hi = E - 1;
  while (lo < hi) {                                  // last expert whose first unit <= unit
    const int mid = (lo + hi + 1) >> 1;
    if (t_unit[mid] <= unit) lo = mid; else hi = mid - 1;
  }
  it.e = lo;
  const int c = unit - t_unit[lo];
  it.nt = min(UT, t_tile[lo + 1] - t_tile[lo] - UT * c);
  it.tile0 = t_tile[lo] + UT * c;
  it.m0 = 0;
  it.m_end = 0;
  if (rows) {
    it.m0 = __ldg(offsets + lo) + static_cast<int64_t>(UT * c) * 128;
    it.m_end = __ldg(offsets + lo + 1);
  }
  return it;
}

// SWI: fused SwiGLU.  An item then runs its K rounds twice, on the gate band n_tile
// (accumulator columns [0, 128)) and on the matching up band n_tile + F/128 (columns
// [128, 256)): virtual rounds 0 .. 2 nr - 1, the second nr on the up band.
template <int FMT, int WSRC, bool SWI>
__global__ void __launch_bounds__(kRoundThreads, 1)
    moe_round_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ MoeRoundParams p) {
  using L = RoundLayout<FMT, WSRC>;
  constexpr int A = L::A, RS = L::RS;
  static_assert(kDecWarps == 16, "decode map assumes 16 decoder warps");

  const int K = p.K, KS = K / kStageK, KB4 = K / L::kB / 4;
  const int n_bands = (SWI ? p.N / 2 : p.N) / kTileN;
  const int qn = p.qn, qk = p.qk;
  const int H = qk == 128 ? 2 : 1;                   // codebooks per stage along K
  const int cb_per_row = K / qk;
  const int nr = (KS + RS - 1) / RS;                 // K rounds
  const int nrv = SWI ? 2 * nr : nr;                 // rounds per item
  auto kr = [&](int v) { return SWI && v >= nr ? v - nr : v; };                     // K round of round v
  auto wband = [&](const RoundItem& it, int v) { return it.n_tile + (SWI && v >= nr ? n_bands : 0); };
  auto qb_first = [&](int ks) { return H == 2 ? 2 * ks : (ks * kStageK) / qk; };
  auto qb_last = [&](int ks) { return H == 2 ? 2 * ks + 1 : (ks * kStageK) / qk; };
  auto qbn_of = [&](int n_tile) { return static_cast<int>((static_cast<int64_t>(n_tile) * 128) / qn); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  // ---- the call's tile and chunk prefixes into shared memory (one round trip) ----
  const int E = p.E;
  int32_t* const t_tile = reinterpret_cast<int32_t*>(smem + L::TAB_OFF);
  int32_t* const t_chunk = t_tile + (E + 1);
  for (int i = static_cast<int>(threadIdx.x); i < 2 * (E + 1); i += kRoundThreads)
    t_tile[i] = i <= E ? p.tile_prefix[i] : p.chunk_prefix[i - (E + 1)];
  __syncthreads();
  const int n_items = n_bands * (SWI ? t_tile[E] : t_chunk[E]);
  const int k_first = blockIdx.x, k_step = gridDim.x;
  if (k_first >= n_items) return;                    // nothing for this CTA
  auto item = [&](int k, bool rows) {
    return round_item<SWI ? 1 : kChunkTiles>(k, n_bands, E, t_tile, t_chunk, p.offsets, rows);
  };

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::CTRL_OFF);
  // A round's weight data comes in two parts: "lo" = its codebooks, scale indices and
  // the index quarters 0-1 of its stages (needed first); "hi" = quarters 2-3 and the
  // direct scale atoms.  The next round's lo (of this item or the next) is requested
  // once the decoders are done with quarter 1, its hi once they are done with quarter 3.
  uint64_t* bar_lo = bars + 0;
  uint64_t* bar_hi = bars + 1;      // [2], by round parity
  uint64_t* bar_x = bars + 3;       // a tile's token operands and scales landed
  uint64_t* dec_ph = bars + 4;      // [2] half h (K-quarters 2h, 2h+1) of the round decoded; half 0 also
                                    //     means (PostScale-QB) the round's weight scales are in TMEM
  uint64_t* xfree = bars + 8;       // MMAs of one (round, tile) done: the token buffer is free
  uint64_t* w_free = bars + 9;      // MMAs of one round's half 0 done: its quarters 0-1 of the operand
                                    //     tiles are free (w_free + 4: half 1, quarters 2-3)
  uint64_t* accum = bars + 10;      // all MMAs of an item done
  uint64_t* acc_free = bars + 11;   // the epilogue (fused SwiGLU: the decoders) has read an item's accumulators
  uint64_t* mma_done = bars + 12;   // every MMA this CTA issued is complete (once, at the end)
  uint64_t* w_free1 = bars + 13;
  uint64_t* sf_ready = bars + 14;   // PreScale+: the round's weight scale atoms are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  constexpr int kBars = 15;
  static_assert(8 * kBars + 4 <= 128, "barriers below the item slots");
  ItemSlot* const slots = reinterpret_cast<ItemSlot*>(smem + L::EXP_OFF);

  // ---- setup ----
  if (warp == 0) {
    if (lane < kBars)
      mbar_init(bars + lane, (lane >= 4 && lane < 6) || lane == 14 ? kDecWarps
                                                                  : lane == 11 ? (SWI ? kDecWarps : kRoundEpiWarps) : 1);
    __syncwarp();
    if (lane == 0) {
      fence_mbar_init();
      prefetch_tensormap(&tmap_x);
    }
  }
  if (warp == 1) {
    __syncwarp();                                    // tcgen05.alloc is warp-aligned
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =============================== loader ===============================
    // the item's expert data into its slot (its first round's copies read it from there)
    auto fill_slot = [&](ItemSlot* sl, const RoundItem& it) {
      sl->w = p.w[it.e];
      sl->qbn[0] = qbn_of(it.n_tile);
      sl->qbn[1] = SWI ? qbn_of(it.n_tile + n_bands) : 0;
    };
    // Each copy is prepared (addresses and byte counts in registers) before the wait
    // that releases it and fired right after: with the decoders keeping the shared
    // memory pipe busy, the loader's own shared-memory reads and address arithmetic
    // take of the order of a thousand SM clocks, which would otherwise sit between
    // the decoders finishing a half and the next round's data being requested.
    struct LoCopy {                                  // a round's first part
      const uint8_t* idx;                            // its index tiles (quarters 0-1 of each stage)
      const uint16_t* cb;                            // its codebooks
      const uint8_t* sidx;                           // PreScale+: its scale-index units
      const uint8_t* scb;                            // PreScale+: the scale codebook (an item's first round)
      uint32_t tx, cb_bytes, sidx_bytes, scb_bytes;
      int rs;
    };
    struct HiCopy {                                  // a round's second part
      const uint8_t* idx;                            // quarters 2-3 of each stage
      const uint8_t* sf;                             // direct scales: the round's scale atoms
      uint32_t tx;
      int rs;
    };
    // The expert weights are read once per (band, chunk) item: evict-first in L2, so
    // that they do not push out the token tiles, which the bands of a chunk share.
    const uint64_t wpol = l2_policy_evict_first();
    auto prepare_lo = [&](const RoundItem& it, int v, const ItemSlot& sl) {    // round v of item it
      const int r = kr(v), band = wband(it, v);
      const int ks0 = r * RS, rs = min(RS, KS - ks0);
      const int qb0 = qb_first(ks0), qb1 = qb_last(ks0 + rs - 1);
      const int qbn = sl.qbn[SWI && v >= nr ? 1 : 0];
      LoCopy c;
      c.rs = rs;
      c.idx = sl.w.idx + (static_cast<size_t>(band) * KS + ks0) * 8192;
      c.cb = sl.w.cb + (static_cast<size_t>(qbn) * cb_per_row + qb0) * 256;
      c.cb_bytes = static_cast<uint32_t>(qb1 - qb0 + 1) * 512;
      c.tx = rs * 4096 + c.cb_bytes;
      c.sidx = nullptr;
      c.scb = nullptr;
      c.sidx_bytes = 0;
      c.scb_bytes = 0;
      if constexpr (L::kSVQ) {
        const SvqGeom sv(sl.w.ds, L::kB, KS);
        c.sidx = sv.unit(sl.w.sidx, band, ks0);
        c.sidx_bytes = static_cast<uint32_t>(((ks0 + rs - 1) >> sv.lspu) - (ks0 >> sv.lspu) + 1) * 128 * sv.G;
        if (v == 0) {
          c.scb = sl.w.scb;
          c.scb_bytes = 256 * sv.ds;
        }
        c.tx += c.sidx_bytes + c.scb_bytes;
      }
      if (r == 0 && lane == 0) {                     // the band's later rounds on their way into L2
        for (int ks = RS; ks < KS; ks += 4)          // 32 KB a request
          l2_prefetch_bulk_hint(sl.w.idx + (static_cast<size_t>(band) * KS + ks) * 8192,
                                static_cast<uint32_t>(min(4, KS - ks)) * 8192, wpol);
        l2_prefetch_bulk(sl.w.cb + static_cast<size_t>(qbn) * cb_per_row * 256,
                         static_cast<uint32_t>(cb_per_row) * 512);
      }
      return c;
    };
    auto fire_lo = [&](const LoCopy& c) {
      mbar_arrive_expect_tx(bar_lo, c.tx);
      for (int s = 0; s < c.rs; ++s)
        bulk_load_hint(smem + L::IDX_OFF + s * 8192, c.idx + s * 8192, 4096, bar_lo, wpol);
      bulk_load(smem + L::CB_OFF, c.cb, c.cb_bytes, bar_lo);
      if constexpr (L::kSVQ) {
        bulk_load(smem + L::SIDX_OFF, c.sidx, c.sidx_bytes, bar_lo);
        if (c.scb_bytes) bulk_load(smem + L::AUX_OFF, c.scb, c.scb_bytes, bar_lo);
      }
    };
    auto prepare_hi = [&](const RoundItem& it, int v, const ItemSlot& sl) {
      const int r = kr(v), band = wband(it, v);
      const int ks0 = r * RS, rs = min(RS, KS - ks0);
      HiCopy c;
      c.rs = rs;
      c.idx = sl.w.idx + (static_cast<size_t>(band) * KS + ks0) * 8192 + 4096;
      c.sf = nullptr;
      c.tx = rs * 4096;
      if constexpr (WSRC == WSRC_VQ_DIRECT) {
        c.sf = sl.w.sf + (static_cast<size_t>(band) * KB4 + static_cast<size_t>(ks0) * A) * 512;
        c.tx += rs * A * 512;
      }
      return c;
    };
    auto fire_hi = [&](const HiCopy& c, int g) {     // g: the global round number
      uint64_t* bar = bar_hi + (g & 1);
      mbar_arrive_expect_tx(bar, c.tx);
      for (int s = 0; s < c.rs; ++s)
        bulk_load_hint(smem + L::IDX_OFF + s * 8192 + 4096, c.idx + s * 8192, 4096, bar, wpol);
      if constexpr (WSRC == WSRC_VQ_DIRECT)
        bulk_load(smem + L::AUX_OFF + (g & 1) * RS * A * 512, c.sf, c.rs * A * 512, bar);
    };
    // The first round of an item into L2 while the item before it runs: its index
    // tiles, codebooks, scale indices and scale codebook, and its first token tile.
    auto prefetch_first_round = [&](const RoundItem& it, const ItemSlot& sl) {
      const int rs = min(RS, KS);
      l2_prefetch_bulk_hint(sl.w.idx + static_cast<size_t>(it.n_tile) * KS * 8192, static_cast<uint32_t>(rs) * 8192,
                            wpol);
      const int qb1 = qb_last(rs - 1);
      l2_prefetch_bulk(sl.w.cb + static_cast<size_t>(sl.qbn[0]) * cb_per_row * 256,
                       static_cast<uint32_t>(qb1 + 1) * 512);
      if constexpr (L::kSVQ) {
        const SvqGeom sv(sl.w.ds, L::kB, KS);
        l2_prefetch_bulk(sv.unit(sl.w.sidx, it.n_tile, 0), static_cast<uint32_t>(sv.U) * 128 * sv.G);
        l2_prefetch_bulk(sl.w.scb, 256 * sv.ds);
      }
      const int64_t rows = it.m_end - it.m0 < 128 ? it.m_end - it.m0 : 128;
      const int boxes = static_cast<int>((rows + kMoeXBox - 1) / kMoeXBox);
      for (int s = 0; s < rs; ++s)
        for (int q = 0; q < boxes; ++q)
          l2_prefetch_tile_2d(&tmap_x, s * 128, static_cast<int>(it.m0) + q * kMoeXBox);
    };
    // Item li's expert data sits in slots[li & 1]: the slot of item li + 1 is filled
    // when item li starts (the decoders read a slot only in the first round of its
    // item, after that round's first part has landed, which the loader requests after
    // filling the slot; by then every reader of the slot's previous item is past it).
    RoundItem cur = item(k_first, true);
    __syncwarp();
    if (elect_one()) fill_slot(&slots[0], cur);
    __syncwarp();
    {
      const LoCopy lo = prepare_lo(cur, 0, slots[0]);
      const HiCopy hi = prepare_hi(cur, 0, slots[0]);
      if (elect_one()) {
        fire_lo(lo);
        fire_hi(hi, 0);
      }
      __syncwarp();
    }
    int nlo = 1, nhi = 1;                            // copies issued so far
    int g = 0;                                       // global round
    bool ok = true;
    for (int k = k_first, li = 0; k < n_items && ok; k += k_step, ++li) {
      const bool has_next = k + k_step < n_items;
      RoundItem nxt = cur;
      ItemSlot& sc = slots[li & 1];
      ItemSlot& sn = slots[(li + 1) & 1];
      if (has_next) {
        nxt = item(k + k_step, true);                // loads in flight while this item runs
        if (elect_one()) {
          fill_slot(&sn, nxt);
          prefetch_first_round(nxt, sn);
        }
        __syncwarp();
      }
      for (int r = 0; r < nrv && ok; ++r, ++g) {
        const bool next_round = r + 1 < nrv || has_next;
        const RoundItem& ni = r + 1 < nrv ? cur : nxt;
        const ItemSlot& ns = r + 1 < nrv ? sc : sn;
        const int nrr = r + 1 < nrv ? r + 1 : 0;
        if (next_round) {
          const LoCopy lo = prepare_lo(ni, nrr, ns);
          const HiCopy hi = prepare_hi(ni, nrr, ns);
          // the decoders are done with this round's codebooks, scale indices and index
          // quarters 0-1: the next round's may come in
          ok = __all_sync(0xffffffffu, mbar_wait(&dec_ph[0], g & 1));
          if (!ok) break;
          if (elect_one()) fire_lo(lo);
          __syncwarp();
          ++nlo;
          // and with quarters 2-3; the direct scale atoms go to the other staging
          // buffer, whose copy to TMEM (round g-1) completed before this round's
          // decode began (the decoders waited for round g-1's MMAs)
          ok = __all_sync(0xffffffffu, mbar_wait(&dec_ph[1], g & 1));
          if (!ok) break;
          if (elect_one()) fire_hi(hi, g + 1);
          __syncwarp();
          ++nhi;
        }
      }
      cur = nxt;
    }
    // Every copy requested lands before the CTA can retire (on the normal path they
    // all have: each was waited for by its consumer).
    if (lane == 0) {
      mbar_wait(bar_lo, (nlo - 1) & 1);
      mbar_wait(bar_hi + ((nhi - 1) & 1), ((nhi - 1) >> 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    bool ok = true;
    int g = 0, kx = 0, i = 0;
    for (int k = k_first; k < n_items && ok; k += k_step, ++i) {
      const RoundItem it = item(k, false);
      for (int v = 0; v < nrv && ok; ++v, ++g) {
        const int r = kr(v);
        const int ks0 = r * RS, rs = min(RS, KS - ks0);
        const uint32_t sfw_c = tmem + L::COL_SFW + (g & 1) * L::SF_COLS;
        if constexpr (!L::kQBS) {
          // the round's weight scale atoms: direct ones as loaded (by round parity),
          // PreScale+ ones once the decoders have built them from the scale indices
          if constexpr (L::kSVQ) ok = __all_sync(0xffffffffu, mbar_wait(sf_ready, g & 1));
          else ok = __all_sync(0xffffffffu, mbar_wait(bar_hi + (g & 1), (g >> 1) & 1));
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t s0 = smem_u32(smem + (L::kSVQ ? L::SFS_OFF : L::AUX_OFF + (g & 1) * RS * A * 512));
            for (int a = 0; a < rs * A; ++a) tc_cp_32x128b_warpx4(sfw_c + 4 * a, sdesc_sf_atom(s0 + a * 512));
          }
          __syncwarp();
        }
        for (int t = 0; t < it.nt && ok; ++t, ++kx) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_x, kx & 1));
          if (!ok) break;
          tc_fence_after();
          const uint32_t sfx_c = tmem + L::COL_SFX + (kx & 1) * L::SF_COLS;
          if (elect_one()) {
            const uint32_t s0 = smem_u32(smem + L::SFX_OFF);
            for (int a = 0; a < rs * A; ++a) tc_cp_32x128b_warpx4(sfx_c + 4 * a, sdesc_sf_atom(s0 + a * 512));
          }
          __syncwarp();
          if (i > 0 && v == 0 && t == 0) {           // the last item's accumulators have been read
            ok = __all_sync(0xffffffffu, mbar_wait(acc_free, (i - 1) & 1));
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t w_s0 = smem_u32(smem + L::W_OFF), x_s0 = smem_u32(smem + L::X_OFF);
          // tile t's accumulator; fused SwiGLU: the gate's, then (second pass) the up's
          const uint32_t d_t = tmem + static_cast<uint32_t>(SWI ? (v >= nr ? 1 : 0) : t) * 128;
          // D[token][channel]: the tokens are the MMA's A operand (M = 128 TMEM lanes),
          // the decoded weight rows its B operand (N = 128 columns), so that each
          // epilogue thread holds one token's row of outputs
          for (int j = 0; j < 4 && ok; ++j) {
            if (t == 0 && (j & 1) == 0) {            // the first tile runs behind the decode
              ok = __all_sync(0xffffffffu, mbar_wait(&dec_ph[j >> 1], g & 1));
              if (!ok) break;
              tc_fence_after();
            }
            if (elect_one()) {
              for (int s = 0; s < rs; ++s) {
                const uint64_t adesc = sdesc_kmajor_sw128(x_s0 + s * 16384 + 32 * j);
                const uint64_t bdesc = sdesc_kmajor_sw128(w_s0 + s * 16384 + 32 * j);
                const uint32_t accf = (r > 0 || s > 0 || j > 0) ? 1u : 0u;
                const uint32_t sfw_t = sfw_c + 4 * s * A, sfx_t = sfx_c + 4 * s * A;
                if constexpr (FMT == FMT_E4M3) {
                  constexpr uint32_t idesc = idesc_mxf4(128, 0, 0, 0);
                  tc_mma_mxf4nvf4_block16(d_t, adesc, bdesc, idesc, sfx_t + 4 * j, sfw_t + 4 * j, accf);
                } else {
                  const int a = j >> 1;
                  const uint32_t id = static_cast<uint32_t>(j & 1) * 2;
                  const uint32_t idesc = idesc_mxf4(128, 1, static_cast<int>(id), static_cast<int>(id));
                  tc_mma_mxf4_block32(d_t, adesc, bdesc, idesc, (sfx_t + 4 * a) | (id << 30),
                                      (sfw_t + 4 * a) | (id << 30), accf);
                }
              }
            }
            __syncwarp();
            if (j == 1 && t == it.nt - 1) {          // quarters 0-1 of the operand tiles may be rewritten
              if (elect_one()) tc_commit(w_free);
              __syncwarp();
            }
          }
          if (!ok) break;
          if (elect_one()) {
            tc_commit(xfree);                        // this tile's token buffer may be refilled
            if (t == it.nt - 1) tc_commit(w_free1);  // and quarters 2-3 of the operand tiles
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (elect_one()) tc_commit(accum);             // the item's accumulators are final
      __syncwarp();
    }
    // our own MMAs finish before the CTA retires
    if (elect_one()) tc_commit(mma_done);
    __syncwarp();
    mbar_wait(mma_done, 0);
  } else if (warp < 2 + kDecWarps) {
    // ============================== decoders ===============================
    const int dw = warp - 2;
    const int s_l = lane & 3;                        // this lane's stage within the round
    // Row of this lane's item, staggered by the stage so that the 8 lanes of a quarter
    // warp read 8 different 16-byte bank groups of the index tiles and write 8
    // different ones of the operand tiles.
    const int row_i = (dw * 8 + (lane >> 2) + 2 * s_l) & 127;
    // Codebook words this lane lays out: entries [16 kb, 16 kb + 16) of its stage's
    // codebook, kb = (dw + s_l/2) mod 16 (over the 16 warps every lane covers all 256
    // entries; the four stages' reads fall in four different bank groups).
    const int kb = (dw + (s_l >> 1)) & 15;
    const int h0 = s_l & 1;
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L::LUT_OFF) + (16 * kb) * 32 + lane;
    const uint32_t lut_lane = smem_u32(smem + L::LUT_OFF) + lane * 4;
    // weight scales: this warp writes the atoms of stage sf_s of each round, in its
    // TMEM lane quadrant
    const int qd = warp & 3, sf_s = dw >> 2;
    auto cb_words = [&](int ks, int epoch, int qb0, uint4* c0, uint4* c1) {
      const int qbk = H == 2 ? 2 * ks + epoch : (ks * kStageK) / qk;
      const uint8_t* cp = smem + L::CB_OFF + (qbk - qb0) * 512 + 32 * kb;
      const uint4 first = *reinterpret_cast<const uint4*>(cp + 16 * h0);
      const uint4 second = *reinterpret_cast<const uint4*>(cp + 16 * (1 - h0));
      *c0 = h0 ? second : first;
      *c1 = h0 ? first : second;
    };
    auto lay_out = [&](bool act, const uint4& a, const uint4& b) {
      if (!act) return;
      const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        lut[(2 * i) * 32] = wv[i] & 0xFFFFu;
        lut[(2 * i + 1) * 32] = wv[i] >> 16;
      }
    };
    int g = 0, di = 0;
    for (int k = k_first; k < n_items; k += k_step, ++di) {
      const RoundItem it = item(k, SWI);
      SvqGeom sv(8, L::kB, KS);                      // the item's, once its first round has landed
      [[maybe_unused]] float w_ts = 1.0f;            // the expert's weight tensor scale
      for (int v = 0; v < nrv; ++v, ++g) {
        const int r = kr(v);
        const int ks0 = r * RS, rs = min(RS, KS - ks0);
        const bool act = s_l < rs;
        const bool sf_act = sf_s < rs;
        const int qb0 = qb_first(ks0);
        // PostScale-QB: the QBlock bytes of this warp's stage, blocks 4a.. (byte a, a < A)
        uint32_t qbs = 0u;
        if constexpr (L::kQBS) {
          const uint8_t* const qbs_row = p.w[it.e].sf + static_cast<size_t>(qbn_of(wband(it, v))) * cb_per_row;
          if (sf_act) {
#pragma unroll
            for (int a = 0; a < A; ++a) {
              const int64_t ch = static_cast<int64_t>(ks0 + sf_s) * kStageK + static_cast<int64_t>(a) * 4 * L::kB;
              qbs |= static_cast<uint32_t>(__ldg(qbs_row + ch / qk)) << (8 * a);
            }
          }
        }
        const bool landed = __all_sync(0xffffffffu, mbar_wait(bar_lo, g & 1));
        if (v == 0) {                                // the item's slot (filled before this copy was requested)
          const ItemSlot& sl = slots[di & 1];
          sv = SvqGeom(sl.w.ds, L::kB, KS);
          w_ts = sl.w.w_tscale;
        }
        uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0, d0 = c0, d1 = c0;
        if (act && landed) {
          cb_words(ks0 + s_l, 0, qb0, &c0, &c1);
          if (H == 2) cb_words(ks0 + s_l, 1, qb0, &d0, &d1);
        }
        if (g > 0) named_bar_sync(2, kDecThreads);  // every lane is done with the last round's copies
        lay_out(act && landed, c0, c1);
        named_bar_sync(2, kDecThreads);              // this round's copies are complete
        // quarters 0-1 of the operand tiles: the last round's MMAs of them are done
        // (and with them the tcgen05.cp of the last round's PreScale+ scale atoms)
        if (g > 0) mbar_wait(w_free, (g - 1) & 1);
        if constexpr (L::kSVQ) {
          // PreScale+ (Table 4 caption: Ks = 256, ds = 8): the round's weight scale atoms
          // in shared memory, each 128-row atom word looked up once from the scale
          // indices and the scale codebook (one word per decoder thread and stage with
          // E4M3-B16); the MMA warp copies them to TMEM with tcgen05.cp
          // Thread dt owns word dt of the A atoms of every stage (atom dt / 128, word
          // dt mod 128 = row (w / 4) + 32 (w mod 4): the SF atom layout); the lookups of
          // all stages are issued before any is stored, so that their shared-memory
          // latencies overlap (one stage after the other they took ~1,500 SM clocks).
          static_assert(128 * A <= kDecThreads, "one atom word per decoder thread and stage");
          const int dt = dw * 32 + lane;
          if (landed && dt < 128 * A) {
            const uint32_t* scb32 = reinterpret_cast<const uint32_t*>(smem + L::AUX_OFF);
            const int word = dt & 127, a = dt >> 7;
            const int r = (word >> 2) + 32 * (word & 3);
            uint32_t wv[RS];
#pragma unroll
            for (int s = 0; s < RS; ++s) {
              const int ks = ks0 + s;
              if (s < rs)
                wv[s] = svq_word(smem + L::SIDX_OFF + ((ks >> sv.lspu) - (ks0 >> sv.lspu)) * 128 * sv.G + r * sv.G, scb32,
                                 sv.lds, sv.kb_base(ks, L::kB) + 4 * a);
            }
#pragma unroll
            for (int s = 0; s < RS; ++s)
              if (s < rs) reinterpret_cast<uint32_t*>(smem + L::SFS_OFF + (s * A + a) * 512)[word] = wv[s];
          }
          fence_proxy_async_smem();                  // atom writes -> tcgen05.cp reads
          __syncwarp();
          if (lane == 0) mbar_arrive(sf_ready);
        }
        // PostScale-QB: weight scale atom a of this warp's stage into TMEM, the QBlock's
        // byte; row `lane` of the atom, column q, holds block scales 4a..4a+3 of weight
        // row 32 q + lane.
        auto sf_atom = [&](int a) {
          if constexpr (L::kQBS) {
            const uint32_t b = ((qbs >> (8 * a)) & 0xFFu) * 0x01010101u;
            tmem_st_32x32b_x4(tmem + (static_cast<uint32_t>(qd * 32) << 16) + L::COL_SFW + (g & 1) * L::SF_COLS +
                                  4 * (sf_s * A + a),
                              make_uint4(b, b, b, b));
          }
        };
        const uint8_t* idx_l = smem + L::IDX_OFF + s_l * 8192 + row_i * 16;
        uint8_t* wt = smem + L::W_OFF + s_l * 16384 + row_i * 128;
        // One K-quarter of this lane's (row, stage) item: 16 index bytes -> 64 FP4 values.
        auto decode_quarter = [&](int j) {
          const uint4 iv = *reinterpret_cast<const uint4*>(idx_l + j * 2048);
          const uint4 o0 = make_uint4(lut32_pair(lut_lane, iv.x, 0), lut32_pair(lut_lane, iv.x, 2),
                                      lut32_pair(lut_lane, iv.y, 0), lut32_pair(lut_lane, iv.y, 2));
          const uint4 o1 = make_uint4(lut32_pair(lut_lane, iv.z, 0), lut32_pair(lut_lane, iv.z, 2),
                                      lut32_pair(lut_lane, iv.w, 0), lut32_pair(lut_lane, iv.w, 2));
          *reinterpret_cast<uint4*>(wt + (((2 * j) ^ (row_i & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(wt + (((2 * j + 1) ^ (row_i & 7)) << 4)) = o1;
        };
        // Half 0: quarters 0-1, with the round's weight scales (before the scale
        // indices and codebook are replaced: the next round's first part comes in after
        // half 0).  Half 1: quarters 2-3.
        for (int h = 0; h < 2; ++h) {
          bool have = landed;
          if (h == 1) {                              // quarters 2-3 of the round's index tiles
            have = mbar_wait(bar_hi + (g & 1), (g >> 1) & 1) && landed;
            if (g > 0) mbar_wait(w_free1, (g - 1) & 1);   // and of the operand tiles, once free
            if (H == 2) {                            // and the stage's second codebook
              named_bar_sync(2, kDecThreads);
              lay_out(act && landed, d0, d1);
              named_bar_sync(2, kDecThreads);
            }
          }
          if constexpr (L::kQBS) {
            if (h == 0) {
              __syncwarp();                          // tcgen05.st is warp-aligned
              if (sf_act) {
#pragma unroll
                for (int a = 0; a < A; ++a) sf_atom(a);
              }
            }
          }
          if (act && have) {
            decode_quarter(2 * h);
            decode_quarter(2 * h + 1);
          }
          if constexpr (L::kQBS) {
            if (h == 0) {
              __syncwarp();
              tmem_st_wait();
              tc_fence_before();
            }
          }
          fence_proxy_async_smem();                  // tile writes -> tensor-core operand reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&dec_ph[h]);
        }
      }
      if constexpr (SWI) {
        // The item's h = SiLU(g) u (gate accumulator columns [0, 128), up [128, 256))
        // for this warp's 32 tokens (its TMEM lane quadrant) and 32 channels, column
        // group dw/4: channels n_tile*128 + 32 (dw/4) .. + 31 of h, in blocks of B.
        // Each block is quantized for the down projection (FP4 codes into h_q, the
        // scale byte into the grouped SF layout); the tile's rows past the expert's
        // get zero scales.
        constexpr int B = L::kB;
        const float scale = w_ts * (p.a_tscale ? *p.a_tscale : 1.0f);
        const float hs = FMT == FMT_E4M3 ? *p.h_tscale : 1.0f;
        const int kbr = p.F / B;
        const int cg = dw >> 2;
        const int64_t q0 = it.m0 + qd * 32;
        const bool live = q0 < it.m_end;             // warp-uniform: some token of the expert here
        const int64_t m = q0 + lane;
        const int64_t srow = static_cast<int64_t>(it.tile0) * 128 + qd * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const bool ep_ok = mbar_wait(accum, di & 1);
        tc_fence_after();
#pragma unroll 1
        for (int c0 = cg * 32; c0 < cg * 32 + 32; c0 += B) {
          float h[B];
          if (live) {
#pragma unroll
            for (int part = 0; part < B / 8; ++part) {   // 8 columns at a time: few live registers
              uint32_t vg[8], vu[8];
              __syncwarp();                          // tcgen05.ld is warp-aligned
              const uint32_t ta = lane_base + c0 + 8 * part;
              tmem_ld_32x32b_x8(ta, vg);
              tmem_ld_32x32b_x8(ta + 128, vu);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 8; ++c)
                h[8 * part + c] = swiglu_fp32(__fmul_rn(__uint_as_float(vg[c]), scale),
                                              __fmul_rn(__uint_as_float(vu[c]), scale));
            }
          }
          if (!ep_ok) continue;
          const int kbh = (it.n_tile * 128 + c0) / B;   // block index along h's channels
          uint32_t sfb = 0u;
          if (live && m < it.m_end) {
            uint32_t q[B / 8];
            quantize_block_f32<B>(h, FMT == FMT_E4M3, hs, q, sfb);
            uint8_t* dst = p.h_q + m * p.ldh + kbh * (B / 2);
            if constexpr (B == 32) *reinterpret_cast<uint4*>(dst) = make_uint4(q[0], q[1], q[2], q[3]);
            else *reinterpret_cast<uint2*>(dst) = make_uint2(q[0], q[1]);
          }
          p.h_sf[sf_offset(srow, kbh, kbr)] = static_cast<uint8_t>(sfb);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);        // the next item's MMAs may overwrite
      }
    }
  } else if (warp < kRoundTokWarp) {
    // ============================== epilogue ==============================
    // Warp 18 + q reads TMEM lane quadrant (18 + q) mod 4: tokens 32 ((18 + q) mod 4)
    // .. + 31 of each tile, each thread one token's 128 output channels of the band.
    const int qd = warp & 3;
    const float a_ts = p.a_tscale ? *p.a_tscale : 1.0f;
    const int out_bf16 = p.out_bf16;
    const int64_t ldy = p.ldy;
    // 16-byte row stores where Y's rows allow them
    const bool vec = (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0 && (ldy % (out_bf16 ? 8 : 4)) == 0;
    int i = 0;
    // (the fused SwiGLU's output is written by the decoder warps)
    for (int k = k_first; k < (SWI ? 0 : n_items); k += k_step, ++i) {
      const RoundItem it = item(k, true);
      const float scale = p.w[it.e].w_tscale * a_ts;
      const bool ep_ok = mbar_wait(accum, i & 1);
      tc_fence_after();
      for (int t = 0; t < it.nt; ++t) {
        const int64_t q0 = it.m0 + static_cast<int64_t>(t) * 128 + qd * 32;   // this warp's first token
        if (q0 >= it.m_end) continue;                // no token of the expert in this quadrant
        const int64_t m = q0 + lane;
        const bool row_ok = ep_ok && m < it.m_end;
        const size_t base = static_cast<size_t>(m) * ldy + static_cast<size_t>(it.n_tile) * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 16) {
          uint32_t v[16];
          __syncwarp();                              // tcgen05.ld is warp-aligned
          tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(qd * 32) << 16) + t * 128 + c0, v);
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
      if (lane == 0) mbar_arrive(acc_free);          // the next item's MMAs may overwrite
    }
  } else {
    // ========================== token-tile loader ==========================
    // The token operands and scales of each (round, tile) of this CTA's items, in the
    // order the MMA warp consumes them, each once the MMAs that read the buffer's
    // previous contents have completed.
    struct XCopy {                                   // one tile's tokens and their scales for one round
      const uint8_t* sf;
      uint32_t tx;
      int ks0, rs, tm0, boxes;
    };
    auto prepare_x = [&](const RoundItem& it, int v, int t) {    // tile t of round v
      XCopy c;
      c.ks0 = kr(v) * RS;
      c.rs = min(RS, KS - c.ks0);
      const int64_t tm0 = it.m0 + static_cast<int64_t>(t) * 128;
      const int64_t rows = it.m_end - tm0 < 128 ? it.m_end - tm0 : 128;
      c.tm0 = static_cast<int>(tm0);
      c.boxes = static_cast<int>((rows + kMoeXBox - 1) / kMoeXBox);
      c.sf = p.a_sf + (static_cast<size_t>(it.tile0 + t) * KB4 + static_cast<size_t>(c.ks0) * A) * 512;
      c.tx = c.rs * c.boxes * kMoeXBox * 128 + c.rs * A * 512;
      return c;
    };
    auto fire_x = [&](const XCopy& c) {
      mbar_arrive_expect_tx(bar_x, c.tx);
      for (int s = 0; s < c.rs; ++s)
        for (int q = 0; q < c.boxes; ++q)
          tma_load_2d(smem + L::X_OFF + s * 16384 + q * kMoeXBox * 128, &tmap_x, (c.ks0 + s) * 128,
                      c.tm0 + q * kMoeXBox, bar_x);
      bulk_load(smem + L::SFX_OFF, c.sf, c.rs * A * 512, bar_x);
    };
    int kx = 0;                                      // (round, tile) copies issued
    bool ok = true;
    for (int k = k_first; k < n_items && ok; k += k_step) {
      const RoundItem it = item(k, true);
      for (int v = 0; v < nrv && ok; ++v) {
        for (int t = 0; t < it.nt && ok; ++t, ++kx) {
          const XCopy xc = prepare_x(it, v, t);
          if (kx > 0) ok = __all_sync(0xffffffffu, mbar_wait(xfree, (kx - 1) & 1));   // the buffer is free
          if (!ok) break;
          if (elect_one()) fire_x(xc);
          __syncwarp();
        }
      }
    }
    // every copy requested lands before the CTA can retire
    if (lane == 0 && kx > 0) mbar_wait(bar_x, (kx - 1) & 1);
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace mxc
