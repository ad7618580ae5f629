// gemv_kernel.cuh -- the decode-shaped MXCode W4A4 linear layer (M <= 16 tokens).
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale", Table 3 (decode
// TPOT): at decode batch sizes the layer streams its weights once, so the time goes
// to bringing the compressed weights in and turning them into tensor-core operands.
// Each CTA owns 128 output channels x a slice of 256-channel stages (split-K over
// the CTAs of a thread-block cluster) and keeps up to 8 stages of it on chip; a
// longer slice (up to 32 stages) runs as rounds of 8 through the same buffers (a
// round's stream is requested once the round before has been multiplied, and goes
// to L2 while that round decodes):
//
//   * the loader copies the slice's index bytes with one 4-D tensor copy per
//     K-quarter (quarter c of every stage: the packed layout stores each 128 x 256
//     tile as four slabs of 64 input channels), quarter 0 first; the MMA warp
//     fetches the round's token tiles with one 3-D tensor copy;
//   * decoder lane l decodes stage l mod 8, so the 32 per-lane codebook copies in
//     shared memory hold, in bank l, the codebook of lane l's stage: the codebooks
//     of the whole slice are laid out once (one entry per 32-bit word, 32 KB) and
//     no lookup meets a bank conflict; two lookups merge with one fixed byte
//     permute;
//   * the decoders finish K-quarter j of every stage before quarter j+1; the MMA
//     warp issues the block-scaled MMAs of quarter j of all stages while quarter
//     j+1 is decoded.  Native FP4 weights use the same quarter-major MMA order, so
//     both give bit-identical results on the same operands;
//   * the index slabs pass through two quarter buffers (quarters 2 and 3 reuse
//     the buffers of quarters 0 and 1 once those are decoded); the weight scale
//     atoms come in by one bulk copy (PostScale-QB: the loader warp builds them
//     from one byte per QBlock) and the MMA warp moves them to TMEM with
//     tcgen05.cp; PreScale+: the loader bulk-copies the round's scale indices
//     (and once the scale codebook) into that staging area and the decoder warps
//     build the atoms from shared memory and write them with tcgen05.st;
//   * token scales: with at most 16 tokens only the first 16 of the 128 rows of
//     an activation scale atom carry scales (the rest is zero padding), so four
//     extra warps, one per TMEM lane quadrant, load those 16 words per atom and
//     write the atoms' TMEM image with tcgen05.st -- the image tcgen05.cp would
//     make of the whole atom -- instead of 144 CTAs copying 16 KB each;
//   * split-K, two ranks, FP32 output: rank 0 zeroes its output tile after the
//     dependency wait (token-scale warps) and both ranks add their scaled partials
//     with red.global.add (two addends onto zero: the result does not depend on
//     their order); more ranks or BF16 output: the partial tiles go to rank 0 as
//     one 8 KB bulk copy between shared memories (completion on an mbarrier there,
//     an acknowledgement back before the sender may exit) and rank 0 adds the
//     scaled partials in rank order (for two ranks the same FP32 value);
//   * split-K through the workspace (more than two ranks, or slices past 8
//     stages, while all CTAs fit one wave and the caller gives the room): no
//     cluster -- a cluster of four one-CTA-per-SM CTAs cannot be placed in one
//     wave -- each
//     rank writes its scaled partial tile to the workspace and takes a ticket from
//     the tile's arrival counter (atomicInc wrapping at splits - 1, so the counter
//     is back at zero after every call); the rank that arrives last adds the
//     partials in rank order, the same FP32 value as the paths above.
//
// Programmatic dependent launch: only the token tiles, the token scales and the
// activation tensor scale come from the previous kernel (typically the activation
// quantizer), and the output tile is written.  Everything else -- loading and
// decoding the whole weight slice, the weight scales into TMEM -- runs before
// griddepcontrol.wait and overlaps that kernel; the MMA warp waits, then fetches
// the token operands, and the decoder warps wait before they touch the output.
// The weight buffers are therefore read while the previous kernel may still run:
// they must not be written by a kernel of the same programmatic-launch chain.
#pragma once

#include "mma_kernel.cuh"

namespace mxc {

constexpr int kGemvT = 16;          // token tile = MMA N
constexpr int kGemvMaxStages = 8;   // 256-channel stages resident per CTA (one round)
constexpr int kGemvMaxRounds = 4;   // rounds per slice: slices of up to 32 stages
constexpr int kGemvMaxSplits = 4;   // cluster size
constexpr int kGemvSfxWarps = 4;    // token-scale warps, one per TMEM lane quadrant
constexpr int kGemvThreads = kThreads + 32 * kGemvSfxWarps;
constexpr int kGemvLutBytes = 256 * 32 * 4;   // 32 per-lane copies, one entry per word

struct GemvParams {
  int M, N, K;
  int qn, qk;                 // resolved QBlock
  const uint8_t* a_sf;        // activation scales, SF layout
  const float* a_tscale;      // device or null
  const float* w_tscale_dev;  // native weights: device tensor scale or null
  void* y;
  int64_t ldy;
  int out_bf16;
  int splits, ks_per_split;
  ExpertPtrs w;
  float* red_part;            // workspace split-K: [tile][rank][128][16] scaled partials, or null
  unsigned int* red_ctr;      // workspace split-K: one arrival counter per output tile (zero on entry)
};

template <int FMT, int WSRC>
struct GemvLayout {
  static constexpr bool kVQ = WSRC != WSRC_NATIVE;
  static constexpr bool kSVQ = WSRC == WSRC_VQ_SVQ;
  static constexpr bool kQBS = WSRC == WSRC_VQ_QBS;   // atoms built from one byte per QBlock
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int kAtoms = kStageK / kB / 4;      // scale atoms per 128 rows per stage
  static constexpr int S = kGemvMaxStages;
  static constexpr int W_OFF = 0;                      // S x [128][128 B] FP4, 128-byte swizzle
  static constexpr int X_OFF = W_OFF + S * 16384;      // S x [16][128 B] FP4 token tiles
  // index slabs, 2 buffers x [S stages][128][16 B] (quarter j in buffer j mod 2).
  // Without the FP32 reduction in global memory, rank 0 receives the other ranks'
  // partial tiles, [rank-1][128][16] FP32, at the start of the index buffers (free
  // once rank 0 has decoded; never used by native weights).
  static constexpr int IDX_OFF = X_OFF + S * kGemvT * 128;
  static constexpr int IDX_BUF = S * 2048;
  // weight scale atoms (direct, native, PostScale-QB); PreScale+: the scale codebook
  // ([256][ds], at most 8 KB) and the round's scale-index units (at most 2 KB)
  static constexpr int SFW_OFF = IDX_OFF + 2 * IDX_BUF;
  static constexpr int SCB_OFF = SFW_OFF;
  static constexpr int SIDX_OFF = SFW_OFF + 8192;
  static constexpr int LUT_OFF = SFW_OFF + (kSVQ ? 16384 : S * kAtoms * 512);   // 256 words x 32 lanes
  static constexpr int CTRL_OFF = LUT_OFF + (kVQ ? kGemvLutBytes : 0);
  // The slice's codebooks (at most 16 x 512 B) land in the second half of the last
  // stage's FP4 tile, which is not written before the codebook copies are laid out.
  static constexpr int CB_OFF = W_OFF + (S - 1) * 16384 + 8192;
  static constexpr int SMEM = 1024 + CTRL_OFF + 256;
  static constexpr int RED = (kGemvMaxSplits - 1) * 128 * kGemvT * 4;
  // TMEM: accumulator [0,16); the scale atoms of all stages, 4 columns each:
  // weight scales from column 32, token scales after them.
  static constexpr int COL_SFW = 32;
  static constexpr int COL_SFX = COL_SFW + S * kAtoms * 4;
  static constexpr int TMEM_COLS = COL_SFX + S * kAtoms * 4 <= 256 ? 256 : 512;
  static_assert(RED <= 2 * IDX_BUF && 128 * kGemvT * 4 <= IDX_BUF, "receive areas");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Writes 8 scale atoms' worth of TMEM columns for this warp's lane quadrant: column 4a
// gets v[a], columns 4a+1..4a+3 get zero (rows 32.. of the atom are padding here).
__device__ __forceinline__ void tmem_st_sfx8(uint32_t taddr, const uint32_t* v) {
  const uint32_t z = 0;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %9, %9, %9, %2, %9, %9, %9, %3, %9, %9, %9, %4, %9, %9, %9, "
      "%5, %9, %9, %9, %6, %9, %9, %9, %7, %9, %9, %9, %8, %9, %9, %9};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(z)
      : "memory");
}
// Two index bytes (k, k+1 of word x) -> 8 FP4 values through this lane's codebook
// copy (lut_lane = copy base + lane*4; entry e in the low half of word e*32 + lane).
__device__ __forceinline__ uint32_t lut32_pair(uint32_t lut_lane, uint32_t x, int k) {
  const uint32_t wa = lds_u32(lut_lane + (((x >> (8 * k)) & 0xFFu) << 7));
  const uint32_t wb = lds_u32(lut_lane + (((x >> (8 * k + 8)) & 0xFFu) << 7));
  return __byte_perm(wa, wb, 0x5410u);
}

// A decoder thread's share of K-quarter j of its lane's stage s_l: two of the stage's
// 128 rows (q and q + 64, offset by the stage so that the 8 stages' stores meet
// different banks), 16 index bytes each from the quarter's slab idx_q, decoded through
// the lane's codebook copy into 32 bytes of row r of the stage tile wt (128-byte
// swizzle: 16-byte chunk c of row r at chunk c ^ (r mod 8)).
__device__ __forceinline__ void decode_quarter_rows(uint32_t lut_lane, const uint8_t* idx_q, uint8_t* wt, int q,
                                                    int s_l, int j) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int rw = (q + 64 * i + s_l) & 127;
    const uint4 iv = *reinterpret_cast<const uint4*>(idx_q + rw * 16);
    const uint4 o0 = make_uint4(lut32_pair(lut_lane, iv.x, 0), lut32_pair(lut_lane, iv.x, 2),
                                lut32_pair(lut_lane, iv.y, 0), lut32_pair(lut_lane, iv.y, 2));
    const uint4 o1 = make_uint4(lut32_pair(lut_lane, iv.z, 0), lut32_pair(lut_lane, iv.z, 2),
                                lut32_pair(lut_lane, iv.w, 0), lut32_pair(lut_lane, iv.w, 2));
    *reinterpret_cast<uint4*>(wt + rw * 128 + (((2 * j) ^ (rw & 7)) << 4)) = o0;
    *reinterpret_cast<uint4*>(wt + rw * 128 + (((2 * j + 1) ^ (rw & 7)) << 4)) = o1;
  }
}

// At most 64 registers a thread (704 x 64 = 45,056 of the SM's 65,536), so that the
// kernel launched next to it (the activation quantizer of the next layer, a
// 16-CTA cluster of 256-thread CTAs) still finds room on the same SMs.
template <int FMT, int WSRC>
__global__ void __maxnreg__(64)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wq,
                const __grid_constant__ CUtensorMap tmap_idx, const __grid_constant__ GemvParams p) {
  using L = GemvLayout<FMT, WSRC>;
  constexpr int A = L::kAtoms;
  static_assert(kDecWarps == 16, "decode map assumes 16 decoder warps");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::CTRL_OFF);
  uint64_t* full = bars;            // [8] VQ: K-quarter j of all index slabs (j < 4); native: stage tiles
  uint64_t* bar_x = bars + 8;       // token tiles
  uint64_t* dec_ph = bars + 9;      // [4] K-quarter j decoded (one arrival per decoder warp)
  uint64_t* sf_ready = bars + 13;   // scale atoms in TMEM (one arrival per decoder warp)
  uint64_t* accum = bars + 14;
  uint64_t* red_full = bars + 15;   // rank 0: partial tiles received
  uint64_t* red_ready = bars + 16;  // rank > 0: rank 0 may receive
  uint64_t* bar_sfw = bars + 17;    // weight scale atoms, or PreScale+ scale indices (+ codebook), by bulk copy
  uint64_t* bar_cb = bars + 18;     // codebooks of the slice (bulk copy)
  uint64_t* sfx_ready = bars + 20; // token scale atoms in TMEM (one arrival per token-scale warp)
  uint64_t* round_free = bars + 21; // a round's MMAs are done: its buffers and scale columns may be reused
  uint64_t* red_ack = bars + 22;    // rank > 0: rank 0 has received this rank's partial tile
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K, KS = K / kStageK, KB4 = K / L::kB / 4;
  const int n_tile = blockIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kGemvT;
  const int sf_group0 = static_cast<int>(m0 / 128);
  const int splits = p.splits;
  const int ks_begin = blockIdx.z * p.ks_per_split;
  const int ks_end = min(KS, ks_begin + p.ks_per_split);
  const int nks = ks_end - ks_begin;
  const bool red_ws = p.red_part != nullptr;                     // split-K through the workspace
  const bool clustered = splits > 1 && !red_ws;                 // the split CTAs of a tile are a cluster
  const uint32_t rank = red_ws ? blockIdx.z : clustered ? cluster_ctarank() : 0u;
  const int H = (L::kVQ && p.qk == 128) ? 2 : 1;     // codebooks per stage along K
  const int qbn = L::kVQ ? static_cast<int>((static_cast<int64_t>(n_tile) * 128) / p.qn) : 0;
  const int cb_per_row = L::kVQ ? K / p.qk : 0;
  // this slice's index tiles: nks contiguous 8 KB tiles, quarter j at +2048 j in each
  const uint8_t* const w_idx = p.w.idx + (static_cast<size_t>(n_tile) * KS + ks_begin) * 8192;
  const uint16_t* const w_cb = p.w.cb + static_cast<size_t>(qbn) * cb_per_row * 256;
  // direct scales: this slice's atoms in the SF layout (PostScale-QB indexes p.w.sf by QBlock)
  const uint8_t* const w_sf = p.w.sf + (static_cast<size_t>(n_tile) * KB4 + static_cast<size_t>(ks_begin) * A) * 512;
  const SvqGeom sv(p.w.ds, L::kB, KS);                // PreScale+ index units of this band
  const uint8_t* const a_sf =
      p.a_sf + (static_cast<size_t>(sf_group0) * KB4 + static_cast<size_t>(ks_begin) * A) * 512;
  const int red_off = L::IDX_OFF;                               // rank 0's receive area
  const bool red_atomic = clustered && splits == 2 && !p.out_bf16;   // split-K by global reductions
  // Slices longer than the 8 resident stages run in rounds of 8: round r covers the
  // stages [ks_begin + 8 r, + rcount(r)).  A round's buffers, TMEM scale columns and
  // token tiles are reused once the MMAs of the round before have completed
  // (round_free); the accumulator runs on across rounds, so the MMAs keep the order
  // round by round, quarter-major within a round.
  const int rounds = (nks + L::S - 1) / L::S;
  const int rbox = min(p.ks_per_split, L::S);         // stages per tensor copy (the maps' box)
  auto rcount = [&](int r) { return min(L::S, nks - L::S * r); };
  // codebooks used by round r: a contiguous range [qb_first, qb_last] of the band's row
  auto qb_first = [&](int r) {
    const int b = ks_begin + L::S * r;
    return !L::kVQ ? 0 : H == 2 ? 2 * b : (b * kStageK) / p.qk;
  };
  auto qb_last = [&](int r) {
    const int e = ks_begin + L::S * r + rcount(r);   // one past the round's last stage
    return !L::kVQ ? 0 : H == 2 ? 2 * e - 1 : ((e - 1) * kStageK) / p.qk;
  };
  // The weight stream of round r, requested at once and in the order it is consumed
  // (nothing here waits for the rest of the CTA or the cluster: the copies land in
  // this CTA's own shared memory on its own barriers).  Codebooks, index quarter 0 of
  // every stage, the weight scales and quarter 1 go straight to shared memory;
  // quarters 2 and 3, whose buffers free up only as quarters 0 and 1 are decoded, go
  // to L2 now and are copied in later.  (A plain L2 prefetch of the slice in address
  // order would complete quarter 0 -- spread over all stages -- only when nearly the
  // whole slice had arrived, and the decode could not overlap it.)
  // Every weight byte is read once per launch: its copies are marked evict-first in
  // L2 (wpol), so that the stream does not evict what each launch reuses -- the kernel
  // code and parameters (whose first reads otherwise go to memory at every launch,
  // ahead of the first copy), the activations and the output.
  const uint64_t wpol = l2_policy_evict_first();
  auto issue_round = [&](int r) {
    const int rb = ks_begin + L::S * r, rn = rcount(r);
    if constexpr (L::kVQ) {
      const int qa = qb_first(r);
      const uint32_t cb_bytes = static_cast<uint32_t>(qb_last(r) - qa + 1) * 512;
      mbar_arrive_expect_tx(bar_cb, cb_bytes);
      bulk_load_hint(smem + L::CB_OFF, w_cb + static_cast<size_t>(qa) * 256, cb_bytes, bar_cb, wpol);
      // quarter j of the round's stages: box {2048 B, 1, rbox stages, 1}; stages past
      // the round (and past K) arrive too, zero-filled past K, and are not used
      mbar_arrive_expect_tx(&full[0], rbox * 2048);
      tma_load_4d_hint(smem + L::IDX_OFF, &tmap_idx, 0, 0, rb, n_tile, &full[0], wpol);
    }
    if constexpr (!L::kSVQ && !L::kQBS) {
      mbar_arrive_expect_tx(bar_sfw, rn * A * 512);
      bulk_load_hint(smem + L::SFW_OFF, w_sf + static_cast<size_t>(L::S * r) * A * 512, rn * A * 512, bar_sfw, wpol);
    }
    if constexpr (L::kVQ) {
      mbar_arrive_expect_tx(&full[1], rbox * 2048);
      tma_load_4d_hint(smem + L::IDX_OFF + L::IDX_BUF, &tmap_idx, 0, 1, rb, n_tile, &full[1], wpol);
      for (int s = 0; s < rn; ++s)
        l2_prefetch_bulk_hint(w_idx + static_cast<size_t>(L::S * r + s) * 8192 + 4096, 4096, wpol);
    } else {
      for (int s = 0; s < rn; ++s) {
        mbar_arrive_expect_tx(&full[s], 16384);
        tma_load_2d_hint(smem + L::W_OFF + s * 16384, &tmap_wq, (rb + s) * 128, n_tile * 128, &full[s], wpol);
      }
    }
    if constexpr (L::kSVQ) {                         // the round's scale indices (+ the scale codebook)
      const int u0 = rb >> sv.lspu, u1 = (rb + rn - 1) >> sv.lspu;
      const uint32_t sidx_bytes = static_cast<uint32_t>(u1 - u0 + 1) * 128 * sv.G;
      const uint32_t scb_bytes = r == 0 ? 256u * static_cast<uint32_t>(sv.ds) : 0u;
      mbar_arrive_expect_tx(bar_sfw, sidx_bytes + scb_bytes);
      bulk_load_hint(smem + L::SIDX_OFF, sv.unit(p.w.sidx, n_tile, rb), sidx_bytes, bar_sfw, wpol);
      if (r == 0) bulk_load(smem + L::SCB_OFF, p.w.scb, scb_bytes, bar_sfw);
    }
  };

  // ---- setup (nothing here depends on earlier kernels) ----
  if (warp == 0) {
    // full[0..7], bar_x, dec_ph[0..3], sf_ready, accum, red_full, red_ready, bar_sfw, bar_cb,
    // (unused), sfx_ready, round_free, red_ack
    if (lane < 23) mbar_init(bars + lane, (lane >= 9 && lane < 14) ? kDecWarps : lane == 20 ? kGemvSfxWarps : 1);
    __syncwarp();
  }
  if (warp == 0 && lane == 0) {
    // rank 0 expects every other rank's partial tile; armed before it lets them send
    if (clustered && rank == 0) mbar_arrive_expect_tx(red_full, (splits - 1) * 128 * kGemvT * 4);
    fence_mbar_init();
    prefetch_tensormap(&tmap_x);
    if constexpr (WSRC == WSRC_NATIVE) prefetch_tensormap(&tmap_wq);
    if constexpr (L::kVQ) prefetch_tensormap(&tmap_idx);
    issue_round(0);                                  // the first round's weight stream
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
  if (clustered) {
    __syncwarp();
    cluster_arrive_relaxed();                        // barriers above are initialised (fenced)
  }
  griddep_launch_dependents();
  if (clustered) {
    __syncwarp();
    cluster_wait_acquire();                          // every CTA of the cluster is set up
  }
  // Two ranks, FP32 output: after the dependency wait rank 0's token-scale warps zero
  // this tile of Y (rows < M) and publish the stores with a release arrive on the
  // second cluster-barrier phase; both ranks then only add to the tile.  All other
  // warps arrive relaxed (a release would wait for their prefetches).  Every
  // cluster-barrier arrive and wait is made by whole, converged warps.
  const bool sfx_warp = warp >= 2 + kDecWarps;
  if (red_atomic && warp < 2) {
    __syncwarp();
    cluster_arrive_relaxed();
  }

  // epilogue coordinates (decoder warps)
  const int qd = warp & 3;                           // TMEM lane quadrant this warp may access
  const int cg = (warp - 2) >> 2;                    // 4-column group of the accumulator
  const int row = qd * 32 + lane;
  const int64_t n = static_cast<int64_t>(n_tile) * 128 + row;
  const int64_t mbase = m0 + cg * 4;

  if (warp == 0) {
    // =============================== loader ===============================
    // (round 0's codebooks, index quarters 0 and 1, weight scales or native weight
    // tiles were requested during setup; the MMA warp fetches the token operands
    // after the dependency wait)
    __syncwarp();
    int last_r = 0;                                  // the last round whose stream was requested
    int issued_q = 2;                                // its index quarters requested so far
    for (int r = 0; r < rounds; ++r) {
      const int rb = ks_begin + L::S * r, rn = rcount(r);
      const uint32_t ph = static_cast<uint32_t>(r & 1);
      if (r > 0) {
        // the round before is multiplied: its buffers take this round's stream
        if (!__all_sync(0xffffffffu, mbar_wait(round_free, (r - 1) & 1))) break;
        if (lane == 0) issue_round(r);
        last_r = r;
        issued_q = 2;
      }
      if constexpr (L::kQBS) {
        // PostScale-QB: the weight scale atoms of the round, each 512 bytes of its
        // QBlock's scale (atoms in the second half of a stage use the second QBlock
        // when the QBlock is 128 wide along K); then the MMA warp copies them to TMEM.
        // Lane i loads atom i's byte (at most 32 atoms), so all loads are in flight at
        // once; each atom then takes its byte from that lane.
        const uint8_t* qb = p.w.sf + static_cast<size_t>((static_cast<int64_t>(n_tile) * 128) / p.qn) * (K / p.qk);
        uint32_t mine = 0;
        if (lane < rn * A) {
          const int ks = rb + lane / A, a = lane % A;
          const int qbk = H == 2 ? 2 * ks + (a >= A / 2 ? 1 : 0) : (ks * kStageK) / p.qk;
          mine = __ldg(qb + qbk);
        }
        for (int i = 0; i < rn * A; ++i) {
          const uint32_t v = __shfl_sync(0xffffffffu, mine, i) * 0x01010101u;
          reinterpret_cast<uint4*>(smem + L::SFW_OFF + i * 512)[lane] = make_uint4(v, v, v, v);
        }
        fence_proxy_async_smem();                    // generic writes -> tcgen05.cp reads
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sfw);
      }
      if constexpr (L::kVQ) {
        if (elect_one()) {
          for (int j = 2; j < 4; ++j) {              // K-quarter j of every stage (from L2 by now)
            if (!mbar_wait(&dec_ph[j - 2], ph)) break;   // its buffer has been decoded
            mbar_arrive_expect_tx(&full[j], rbox * 2048);
            tma_load_4d_hint(smem + L::IDX_OFF + (j % 2) * L::IDX_BUF, &tmap_idx, 0, j, rb, n_tile, &full[j], wpol);
            issued_q = j + 1;
          }
          if (issued_q == 4 && r + 1 < rounds) {     // the next round's stream into L2 meanwhile
            const int nb = L::S * (r + 1), nn = rcount(r + 1);
            l2_prefetch_bulk_hint(w_idx + static_cast<size_t>(nb) * 8192, static_cast<uint32_t>(nn) * 8192, wpol);
            if constexpr (!L::kSVQ && !L::kQBS)
              l2_prefetch_bulk_hint(w_sf + static_cast<size_t>(nb) * A * 512, static_cast<uint32_t>(nn) * A * 512,
                                    wpol);
            if constexpr (L::kSVQ) {
              const int nbs = ks_begin + nb;
              const int u0 = nbs >> sv.lspu, u1 = (nbs + nn - 1) >> sv.lspu;
              l2_prefetch_bulk(sv.unit(p.w.sidx, n_tile, nbs), static_cast<uint32_t>(u1 - u0 + 1) * 128 * sv.G);
            }
          }
        }
        issued_q = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(issued_q)));   // the elected lane's count
      }
      __syncwarp();
    }
    // Every copy this CTA requested lands before the CTA can retire, even when a
    // consumer gave up waiting (timeout path): codebooks, index quarters, weight
    // scales or native tiles.  The copies of earlier rounds completed before their
    // round's MMAs did; on the normal path the last round's have completed too.
    if (lane == 0) {
      const uint32_t ph = static_cast<uint32_t>(last_r & 1);
      if constexpr (L::kVQ) {
        mbar_wait(bar_cb, ph);
        for (int j = 0; j < issued_q; ++j) mbar_wait(&full[j], ph);
      } else {
        for (int s = 0; s < rcount(last_r); ++s) mbar_wait(&full[s], ph);
      }
      if constexpr (!L::kQBS) mbar_wait(bar_sfw, ph);
    }
    __syncwarp();
    if (clustered && rank == 0 && !red_atomic) {
      // Let the other ranks send their partials once the receive area (the index
      // buffers) is free: after the last decode phase.  Sent even after a failed
      // wait, so that no rank waits for the signal in vain.
      if constexpr (L::kVQ) mbar_wait(&dec_ph[3], static_cast<uint32_t>((rounds - 1) & 1));
      if (lane > 0 && lane < splits) mbar_remote_arrive(mapa_shared(smem_u32(red_ready), lane));
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    const uint32_t w_s0 = smem_u32(smem + L::W_OFF), x_s0 = smem_u32(smem + L::X_OFF);
    bool ok = true;
    for (int r = 0; r < rounds && ok; ++r) {
      const int rb = ks_begin + L::S * r, rn = rcount(r);
      const uint32_t ph = static_cast<uint32_t>(r & 1);
      if (r > 0) {                                   // the round before has been multiplied
        ok = __all_sync(0xffffffffu, mbar_wait(round_free, (r - 1) & 1));
        if (!ok) break;
        tc_fence_after();
      }
      if constexpr (!L::kSVQ) {
        // weight scale atoms -> TMEM; copies and MMAs issue in order from this thread
        ok = __all_sync(0xffffffffu, mbar_wait(bar_sfw, ph));
        if (ok && elect_one()) {
          const uint32_t sfw_s0 = smem_u32(smem + L::SFW_OFF);
          for (int i = 0; i < rn * A; ++i)
            tc_cp_32x128b_warpx4(tmem + L::COL_SFW + 4 * i, sdesc_sf_atom(sfw_s0 + i * 512));
        }
        __syncwarp();
      }
      if (r == 0) griddep_wait();                    // the token operands are written
      __syncwarp();
      if (elect_one()) {
        // token tiles of the round's stages: box {128 B, 16 rows, rbox stages}; stages
        // past the round (and past K) arrive too, zero-filled past K, and are not used
        mbar_arrive_expect_tx(bar_x, rbox * kGemvT * 128);
        tma_load_3d(smem + L::X_OFF, &tmap_x, 0, static_cast<int>(m0), rb, bar_x);
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, mbar_wait(sfx_ready, ph)) && ok;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_x, ph)) && ok;
      if constexpr (L::kSVQ) ok = __all_sync(0xffffffffu, mbar_wait(sf_ready, ph)) && ok;
      if constexpr (!L::kVQ) {
        for (int s = 0; s < rn && ok; ++s) ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph));
      }
      tc_fence_after();
      for (int j = 0; j < 4 && ok; ++j) {
        if constexpr (L::kVQ) {
          if (!__all_sync(0xffffffffu, mbar_wait(&dec_ph[j], ph))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (elect_one()) {
          for (int s = 0; s < rn; ++s) {
            const uint64_t adesc = sdesc_kmajor_sw128(w_s0 + s * 16384 + 32 * j);
            const uint64_t bdesc = sdesc_kmajor_sw128(x_s0 + s * kGemvT * 128 + 32 * j);
            const uint32_t acc = (r > 0 || s > 0 || j > 0) ? 1u : 0u;
            const uint32_t sfw_t = tmem + L::COL_SFW + 4 * s * A, sfx_t = tmem + L::COL_SFX + 4 * s * A;
            if constexpr (FMT == FMT_E4M3) {
              constexpr uint32_t idesc = idesc_mxf4(kGemvT, 0, 0, 0);
              tc_mma_mxf4nvf4_block16(tmem, adesc, bdesc, idesc, sfw_t + 4 * j, sfx_t + 4 * j, acc);
            } else {
              const int a = j >> 1;
              const uint32_t id = static_cast<uint32_t>(j & 1) * 2;
              const uint32_t idesc = idesc_mxf4(kGemvT, 1, static_cast<int>(id), static_cast<int>(id));
              tc_mma_mxf4_block32(tmem, adesc, bdesc, idesc, (sfw_t + 4 * a) | (id << 30),
                                  (sfx_t + 4 * a) | (id << 30), acc);
            }
          }
        }
        __syncwarp();
      }
      if (ok && r + 1 < rounds && elect_one()) tc_commit(round_free);   // the round's buffers may be refilled
      __syncwarp();
    }
    if (elect_one()) tc_commit(accum);
    __syncwarp();
    mbar_wait(accum, 0);      // our own MMAs finish before the CTA retires
  } else if (sfx_warp) {
    // ========================= token scales -> TMEM =========================
    // Row r < 16 of atom i is word r of the atom's first 16 lines (line r, bytes
    // 0..3 of 16); tcgen05.cp of the whole atom would put line l into lane l of
    // every lane quadrant, columns 4i..4i+3.  Rows 16..127 are zero padding.
    griddep_wait();                                  // the activation scales are written
    // Lane l < 16 loads row l of atoms 0..15, lane l + 16 row l of atoms 16..31 (all
    // loads in flight at once); the upper half reaches lanes 0..15 by a shuffle.
    const uint32_t taddr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + L::COL_SFX;
    const int r16 = lane & 15, half = lane >> 4;
    for (int r = 0; r < rounds; ++r) {
      const int na = rcount(r) * A;                  // the round's atoms
      const uint8_t* const a_sf_r = a_sf + static_cast<size_t>(L::S * r) * A * 512;
      if (r > 0) {                                   // the round before has been multiplied
        if (!__all_sync(0xffffffffu, mbar_wait(round_free, (r - 1) & 1))) break;
        tc_fence_after();
      }
      uint32_t v[16];
#pragma unroll
      for (int a = 0; a < 16; ++a) {
        const int atom = 16 * half + a;
        v[a] = atom < na
                   ? __ldg(reinterpret_cast<const uint32_t*>(a_sf_r + static_cast<size_t>(atom) * 512 + r16 * 16))
                   : 0u;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {                  // 8 atoms = 32 columns per store
        if (8 * c >= na) break;                      // uniform over the warp
        uint32_t w[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const uint32_t x = c < 2 ? v[8 * c + a] : __shfl_down_sync(0xffffffffu, v[8 * (c - 2) + a], 16);
          w[a] = half == 0 ? x : 0u;                 // lanes 16..31: padding rows
        }
        __syncwarp();                                // tcgen05.st is warp-aligned
        tmem_st_sfx8(taddr + 32 * c, w);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sfx_ready);
    }
    if (red_atomic) {
      if (rank == 0) {                               // zero this tile of Y, rows < M
        const int st = threadIdx.x - (2 + kDecWarps) * 32;
        for (int e = st; e < kGemvT * 128; e += 32 * kGemvSfxWarps) {
          const int64_t m = m0 + e / 128;
          if (m < p.M) reinterpret_cast<float*>(p.y)[m * p.ldy + static_cast<int64_t>(n_tile) * 128 + (e & 127)] = 0.0f;
        }
      }
      __syncwarp();
      if (rank == 0) cluster_arrive_release(); else cluster_arrive_relaxed();
    }
  } else {
    // ======================= decoders, then epilogue ======================
    const int dw = warp - 2;
    // --- the stage codebook words this lane lays out (loads issued first) ---
    const int s_l = lane & 7;                        // this lane's stage
    const int q = dw * 4 + (lane >> 3);              // 64 threads per stage
    // Entries [16 kb, 16 kb + 16) of the codebook of this lane's stage (first or,
    // QBlock 128 wide along K, second half of the stage), kb = (dw + s_l/2) mod 16:
    // over the 16 warps each lane still covers all 256 entries, and the 8 lanes of a
    // quarter warp (8 stages, codebooks 512 B apart) read 8 different bank groups --
    // the two 16-byte halves are read in an order that alternates with the stage.
    const int kb = (dw + (s_l >> 1)) & 15;
    const int h0 = s_l & 1;
    auto cb_words = [&](int r, int epoch, uint4* c0, uint4* c1) {
      const int ks = ks_begin + L::S * r + s_l;
      const int qbk = H == 2 ? 2 * ks + epoch : (ks * kStageK) / p.qk;
      const uint8_t* cp = smem + L::CB_OFF + (qbk - qb_first(r)) * 512 + 32 * kb;
      const uint4 first = *reinterpret_cast<const uint4*>(cp + 16 * h0);
      const uint4 second = *reinterpret_cast<const uint4*>(cp + 16 * (1 - h0));
      *c0 = h0 ? second : first;                      // entries 16 kb .. 16 kb + 7
      *c1 = h0 ? first : second;                      // entries 16 kb + 8 .. 16 kb + 15
    };

    // --- PreScale+ weight scale atoms -> TMEM lanes of this warp's quadrant
    //     (atoms i = cg mod 4), after decode phase 0 ---
    auto svq_scales_to_tmem = [&](int r) {
      if constexpr (L::kSVQ) {
        __syncwarp();                                // tcgen05.st is warp-aligned
        // PreScale+ (Table 4 caption: Ks = 256, ds = 8; larger ds compress further):
        // row `lane` of atom (s, a) holds, for rows 32 g + lane (g = 0..3), block
        // scales 4a..4a+3 of stage s: one word of the scale-codebook entry.  The
        // round's scale indices and the scale codebook are in shared memory.
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const bool have = mbar_wait(bar_sfw, static_cast<uint32_t>(r & 1));
        const uint32_t* scb32 = reinterpret_cast<const uint32_t*>(smem + L::SCB_OFF);
        const int u0 = (ks_begin + L::S * r) >> sv.lspu;
        for (int i = cg; i < rcount(r) * A; i += 4) {
          const int s = i / A, a = i % A;
          const int ks = ks_begin + L::S * r + s;
          const uint8_t* un = smem + L::SIDX_OFF + ((ks >> sv.lspu) - u0) * 128 * sv.G;
          const int kb = sv.kb_base(ks, L::kB) + 4 * a;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (have) {
            v.x = svq_word(un + (0 * 32 + lane) * sv.G, scb32, sv.lds, kb);
            v.y = svq_word(un + (1 * 32 + lane) * sv.G, scb32, sv.lds, kb);
            v.z = svq_word(un + (2 * 32 + lane) * sv.G, scb32, sv.lds, kb);
            v.w = svq_word(un + (3 * 32 + lane) * sv.G, scb32, sv.lds, kb);
          }
          tmem_st_32x32b_x4(lane_base + L::COL_SFW + 4 * i, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_ready);
      }
    };

    if constexpr (L::kVQ) {
      uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L::LUT_OFF) + (16 * kb) * 32 + lane;
      const uint32_t lut_lane = smem_u32(smem + L::LUT_OFF) + lane * 4;
      const uint8_t* idx_l = smem + L::IDX_OFF + s_l * 2048;
      uint8_t* wt = smem + L::W_OFF + s_l * 16384;
      for (int r = 0; r < rounds; ++r) {
        const uint32_t ph = static_cast<uint32_t>(r & 1);
        const bool active = s_l < rcount(r);
        // both codebooks into registers now: the staging area is overwritten by the
        // decoded tiles of the last stage.  (Every decoder is done with the copies of
        // the round before: its MMAs, which waited for all decode phases, completed
        // before this round's codebooks were requested.)
        uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0, d0 = c0, d1 = c0;
        const bool cb_ok = mbar_wait(bar_cb, ph);
        if (active && cb_ok) {
          cb_words(r, 0, &c0, &c1);
          if (H == 2) cb_words(r, 1, &d0, &d1);
        }
        // --- codebook copies: lane l's copy (bank l) = codebook of stage l mod 8,
        //     entry e in the low half of word e*32 + l ---
        auto lay_out = [&](const uint4& a, const uint4& b) {
          if (!active) return;
          const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            lut[(2 * i) * 32] = w[i] & 0xFFFFu;
            lut[(2 * i + 1) * 32] = w[i] >> 16;
          }
        };
        lay_out(c0, c1);
        named_bar_sync(2, kDecThreads);              // all copies written
        for (int j = 0; j < 4; ++j) {
          if (H == 2 && j == 2) {                    // second half of each stage: its own codebook
            named_bar_sync(2, kDecThreads);          // everyone is done with the first codebooks
            lay_out(d0, d1);
            named_bar_sync(2, kDecThreads);
          }
          const bool landed = mbar_wait(&full[j], ph);
          if (active && landed) decode_quarter_rows(lut_lane, idx_l + (j % 2) * L::IDX_BUF, wt, q, s_l, j);
          fence_proxy_async_smem();                  // tile writes -> tensor-core operand reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&dec_ph[j]);
          if (j == 0) svq_scales_to_tmem(r);         // needed with quarter 0's MMAs
        }
      }
    }
    // ------------------------------ epilogue ------------------------------
    __syncwarp();
    griddep_wait();                                  // the output and the token scale may be touched
    if (red_atomic) {
      __syncwarp();
      cluster_arrive_relaxed();
    }
    float out_scale = p.w.w_tscale;
    if constexpr (WSRC == WSRC_NATIVE) {
      if (p.w_tscale_dev) out_scale = __ldg(p.w_tscale_dev);
    }
    if (p.a_tscale) out_scale *= __ldg(p.a_tscale);
    const bool ep_ok = mbar_wait(accum, 0);
    tc_fence_after();
    const float scale = out_scale;
    uint32_t acc[4];
    __syncwarp();                                    // tcgen05.ld is warp-aligned: converge after the waits
    tmem_ld_32x32b_x4(tmem + (static_cast<uint32_t>(qd * 32) << 16) + cg * 4, acc);
    tmem_ld_wait();
    float v[4] = {__uint_as_float(acc[0]), __uint_as_float(acc[1]), __uint_as_float(acc[2]), __uint_as_float(acc[3])};
    bool store = ep_ok;
    if (red_atomic) {
      store = false;
      __syncwarp();
      cluster_wait_acquire();                        // rank 0's zeroing is visible
      if (ep_ok) {
        float* const y = reinterpret_cast<float*>(p.y);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (mbase + c < p.M) atomicAdd(y + (mbase + c) * p.ldy + n, __fmul_rn(v[c], scale));
      }
    } else if (red_ws) {
      // the scaled partial into this rank's slot; the last rank to arrive at the
      // tile's counter adds all partials in rank order (products and sums rounded
      // separately, no fused multiply-add: the value of the other split-K paths)
      store = false;
      const size_t tile = static_cast<size_t>(blockIdx.y) * gridDim.x + n_tile;
      float* const part = p.red_part + tile * splits * (128 * kGemvT);
      const int off = row * kGemvT + cg * 4;
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = __fmul_rn(v[c], scale);
      const float4 own = make_float4(v[0], v[1], v[2], v[3]);
      __stcg(reinterpret_cast<float4*>(part + static_cast<size_t>(rank) * (128 * kGemvT) + off), own);
      __threadfence();                               // the partial is visible before the ticket
      named_bar_sync(2, kDecThreads);
      uint32_t* const last = reinterpret_cast<uint32_t*>(bars + 25);
      if (threadIdx.x == 64)                         // every CTA arrives once, also after a failed wait
        *last = atomicInc(p.red_ctr + tile, static_cast<unsigned>(splits - 1)) == static_cast<unsigned>(splits - 1);
      named_bar_sync(2, kDecThreads);
      if (*last) {
        __threadfence();                             // the other ranks' partials are visible
        float4 a = rank == 0 ? own : __ldcg(reinterpret_cast<const float4*>(part + off));
        for (int r = 1; r < splits; ++r) {
          const float4 o = r == static_cast<int>(rank)
                               ? own
                               : __ldcg(reinterpret_cast<const float4*>(part + static_cast<size_t>(r) * (128 * kGemvT) + off));
          a.x = __fadd_rn(a.x, o.x);
          a.y = __fadd_rn(a.y, o.y);
          a.z = __fadd_rn(a.z, o.z);
          a.w = __fadd_rn(a.w, o.w);
        }
        v[0] = a.x;
        v[1] = a.y;
        v[2] = a.z;
        v[3] = a.w;
        store = ep_ok;
      }
    } else if (splits > 1) {
      if (rank != 0) {
        // the partial tile [128][16] FP32 into this CTA's receive-area offset, then one
        // bulk copy to rank 0's slot rank-1 (sent even when ep_ok is false: rank 0 waits)
        store = false;
        *reinterpret_cast<float4*>(smem + red_off + (row * kGemvT + cg * 4) * 4) = make_float4(v[0], v[1], v[2], v[3]);
        fence_proxy_async_smem();                    // generic writes -> the bulk copy's reads
        named_bar_sync(2, kDecThreads);
        if (threadIdx.x == 64) {
          if (mbar_wait(red_ready, 0)) {
            constexpr uint32_t kTile = 128 * kGemvT * 4;
            bulk_copy_to_cluster(mapa_shared(smem_u32(smem + red_off) + (rank - 1) * kTile, 0),
                                 smem_u32(smem + red_off), kTile, mapa_shared(smem_u32(red_full), 0));
          }
          // rank 0 has it (or gave up waiting): the source may go.  Rank 0 always sends
          // this acknowledgement, so no rank exits while rank 0 still signals it.
          mbar_wait(red_ack, 0);
        }
      } else {
        const bool got = mbar_wait(red_full, 0);    // all partials landed: none in flight at exit
        if (threadIdx.x == 64) {                     // let the senders go
          for (uint32_t r = 1; r < static_cast<uint32_t>(splits); ++r)
            mbar_remote_arrive(mapa_shared(smem_u32(red_ack), r));
        }
        store = store && got;
        if (store) {
          // scaled partials summed in rank order: with two ranks the same FP32 value
          // as the reduction in global memory (+0 + s*v0 + s*v1), so a BF16 output is
          // exactly the rounding of the FP32 one
          // (separately rounded products and sums: no contraction into an FMA)
#pragma unroll
          for (int c = 0; c < 4; ++c) v[c] = __fmul_rn(v[c], scale);
          for (int r = 1; r < splits; ++r) {
            const float4 o = *reinterpret_cast<const float4*>(smem + red_off + ((r - 1) * 128 * kGemvT +
                                                                                  row * kGemvT + cg * 4) * 4);
            v[0] = __fadd_rn(v[0], __fmul_rn(o.x, scale));
            v[1] = __fadd_rn(v[1], __fmul_rn(o.y, scale));
            v[2] = __fadd_rn(v[2], __fmul_rn(o.z, scale));
            v[3] = __fadd_rn(v[3], __fmul_rn(o.w, scale));
          }
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = __fmul_rn(v[c], scale);   // no split: scale the whole sum
    }
    if (store) {
      void* const y = p.y;
      const int64_t ldy = p.ldy;
      const int out_bf16 = p.out_bf16;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (mbase + c < p.M) store_out(y, ldy, out_bf16, mbase + c, n, v[c]);
    }
  }
  if (red_atomic && (warp < 2 || sfx_warp)) {        // every thread completes the barrier phase
    __syncwarp();
    cluster_wait_acquire();
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
