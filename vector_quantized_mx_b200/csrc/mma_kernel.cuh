// mma_kernel.cuh -- the MXCode W4A4 linear layer on sm_100a tensor cores.
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale" (abstract): the
// VQ storage is turned directly into MX-native W4A4 operands, and no
// high-precision copy of the weight is ever formed.  Here every CTA owns a
// 128 (output channels) x T (tokens) tile of Y^T and runs a pipeline over K in
// stages of 256 input channels:
//
//   warp 0      loader: TMA of the token tile (FP4, 128-byte swizzle) and bulk
//               copies of its scale atoms, the stage's packed index tile (8 KB),
//               its QBlock codebook(s) (512 B each) and the weight scales (direct
//               atoms, or scale-VQ indices).  Native FP4 weights come by TMA.
//   warps 2..17 decoders (two groups of 8 warps on alternate stages for T <= 128,
//               all 16 on every stage for T = 256): the stage's codebook is
//               replicated once per lane (so the random gathers are free of bank
//               conflicts), then every index becomes a 16-bit codebook entry (4
//               E2M1 codes) and 16-byte chunks of FP4 are written straight into
//               the swizzled K-major operand tile the tensor core reads.  PreScale+
//               scale indices become scale bytes in the tcgen05 scale-factor atom
//               layout; PostScale-QB atoms are filled with the QBlock's scale byte.
//               Then epilogue.
//   warp 1      one thread issues tcgen05.cp (scale atoms -> TMEM) and four
//               tcgen05.mma block-scaled FP4 MMAs (K = 64 each) per stage into a
//               128 x T FP32 accumulator in TMEM, and frees the stage with
//               tcgen05.commit.
//   epilogue    warps 2..17 read the accumulator with tcgen05.ld, apply the FP32
//               tensor scales and store FP32/BF16 rows of Y.  For split-K (decode)
//               the CTAs of one output tile form a thread-block cluster: ranks
//               1.. write their partial tiles into rank 0's shared memory and
//               rank 0 adds them in rank order (deterministic, no workspace).
//
// The weight tile is the MMA's A operand (M = 128 rows of W), the token tile is
// the B operand (N = T tokens), so one kernel serves the decode shapes the decode
// GEMV does not take (T = 16) and prefill (T = 128 or 256) without a transpose.
#pragma once

#include "act_quant.cuh"
#include "mxc_device.cuh"
#include "mxc_internal.h"

namespace mxc {

// Weight sources: VQ with block scales stored directly, VQ with VQ-coded block
// scales (PreScale+), native FP4, VQ with one scale per QBlock (PostScale-QB).
enum : int { WSRC_VQ_DIRECT = 0, WSRC_VQ_SVQ = 1, WSRC_NATIVE = 2, WSRC_VQ_QBS = 3 };
enum : int { FMT_E8M0 = 0, FMT_E4M3 = 1 };

constexpr int kMaxSplits = 4;      // cluster split-K factor of the decode path
constexpr int kMoeXBox = 32;       // rows per token-tile copy of an expert tile

struct ExpertPtrs {
  const uint8_t* idx;
  const uint16_t* cb;
  const uint8_t* sf;     // weight scales: SF layout (VQ direct, native)
  const uint8_t* sidx;   // PreScale+ scale indices (packed tiles)
  const uint8_t* scb;    // PreScale+ scale codebook [256][8]
  float w_tscale;
  int ds;                // PreScale+ scale group (block scales per scale index)
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
  int splits, ks_per_split;  // split-K over a cluster of `splits` CTAs (1 = off), or through the workspace
  float* red_part;           // 128-token tiles, split-K through the workspace: [tile][rank][T][128] scaled
                             // partials, or null
  unsigned int* red_ctr;     // and one arrival counter per output tile (zero on entry, zero again at exit)
  ExpertPtrs w[NEXP];
};

// Shared-memory layout of one pipeline stage and of the whole CTA.  NCB = codebooks
// per 256-channel stage: 2 when the QBlock is 128 wide along K, else 1.
template <int FMT, int WSRC, int T, int NCB = 1>
struct StageLayout {
  static constexpr bool kVQ = WSRC != WSRC_NATIVE;
  static constexpr bool kSVQ = WSRC == WSRC_VQ_SVQ;
  static constexpr bool kQBS = WSRC == WSRC_VQ_QBS;
  static constexpr bool kSfwDec = kSVQ || kQBS;       // weight scale atoms written by the decoders
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int kAtoms = kStageK / kB / 4;     // scale atoms per 128 rows per stage
  static constexpr int kXG = (T + 127) / 128;         // 128-row scale groups in the token tile
  static constexpr int kG = kStageK / (8 * kB);       // PreScale+ index bytes per row per stage, at most
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
  static constexpr int LUT = kVQ ? 2 * NCB * 128 * 32 * 4 : 0;       // 2 buffers of per-lane codebook copies
  static constexpr int RED = T <= 32 ? (kMaxSplits - 1) * T * 128 * 4 : 0;  // split-K receive slots
  static constexpr int BUDGET = 227 * 1024 - 1024 - CTRL - LUT - RED;
  static constexpr int STAGES = (BUDGET / BYTES) > 8 ? 8 : (BUDGET / BYTES);
  static constexpr int LUT_OFF = CTRL + STAGES * BYTES;
  static constexpr int RED_OFF = LUT_OFF + LUT;
  static constexpr int SMEM = 1024 + RED_OFF + RED;
  // TMEM columns: accumulator [0, T), weight scales [T, T+16), token scales after.
  static constexpr int COL_SFW = T;
  static constexpr int COL_SFX = T + 16;
  static constexpr int COLS_USED = T + 16 + 16 * kXG;
  static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                   : COLS_USED <= 256 ? 256 : 512;
  static_assert(STAGES >= 2, "stage does not fit");
  static_assert(T % 16 == 0 && T >= 16 && T <= 256, "token tile");
  static_assert(SMEM <= 232448, "shared memory");
};

#ifndef MXC_DEC_WARPS
#define MXC_DEC_WARPS 16
#endif
constexpr int kDecWarps = MXC_DEC_WARPS;           // decoder / epilogue warps (4 per SM sub-partition)
constexpr int kColGroups = kDecWarps / 4;          // epilogue warps per TMEM lane quadrant
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kThreads = 64 + kDecThreads;         // + loader warp + MMA warp

// Decoder groups: with token tiles of up to 128 the tensor-core work per stage is
// short, so two groups of 8 warps decode alternate stages at the same time (each
// with its own codebook copies and named barrier); with 256 one group decodes
// every stage with double-buffered copies.
template <int T>
__host__ __device__ constexpr int dec_groups() { return T <= 128 ? 2 : 1; }

// ------------------------------------------------------------------------------------
// Decoders (shared with the decode-dump kernel).  dt = decoder thread 0..NT-1.
// ------------------------------------------------------------------------------------
// Per-lane codebook copies with 16-bit entries: word (j*32 + lane) holds centroids
// 2j (low half) and 2j+1 (high half), so the 32 lanes of a warp always read 32
// different banks.  `ncb` = 1 or 2 codebooks (two when the QBlock is 128 wide along
// K), 16 KB each.  Stores are 16 B per thread over consecutive addresses (bank-
// conflict free).
constexpr int kLutBytes = 128 * 32 * 4;
template <int NT>
__device__ __forceinline__ void build_lut(const uint16_t* __restrict__ cb, int ncb, uint32_t* __restrict__ lut,
                                          int dt) {
  const uint32_t* cb32 = reinterpret_cast<const uint32_t*>(cb);
  for (int u = dt; u < 1024 * ncb; u += NT) {   // uint4 u: words 4u..4u+3 = entry word u/8, lanes 4(u%8)..
    const uint32_t v = cb32[u >> 3];
    reinterpret_cast<uint4*>(lut)[u] = make_uint4(v, v, v, v);
  }
}

// Two index bytes (k, k+1 of word x) -> 8 FP4 values (32 bits) through this lane's
// codebook copy (lut_lane = copy base + lane*4): the word (e/2)*32 + lane holds
// entry e in half e%2; one byte permute merges both lookups, its selector picking
// each entry's half.
__device__ __forceinline__ uint32_t lut16_pair(uint32_t lut_lane, uint32_t x, int k) {
  const uint32_t wa = lds_u32(lut_lane + (((x >> (8 * k + 1)) & 0x7Fu) << 7));
  const uint32_t wb = lds_u32(lut_lane + (((x >> (8 * k + 9)) & 0x7Fu) << 7));
  return __byte_perm(wa, wb, 0x5410u + ((x >> (8 * k)) & 0x101u) * 0x22u);
}

// One 128 x 256 weight tile: idx (four K-quarter slabs [128][16] bytes) -> FP4
// [128][128] bytes in the 128-byte swizzle (16-byte chunk j of row r stored at
// chunk j ^ (r % 8)).  Item (r, q) = the 16 indices of row r in quarter q -> FP4
// chunks 2q, 2q+1 of row r.  Thread dt owns items it*NT + dt, r = item % 128, so
// the lanes of a warp read consecutive rows of one slab (16-byte loads, no bank
// conflict) and store to 8 different bank groups per quarter warp.  Offsets are
// fixed per thread and computed once (ItemMap).  Quarters 2, 3 use codebook 1 when
// the QBlock is 128 wide along K.
template <int NT>
struct ItemMap {
  static constexpr int kN = 512 / NT;
  uint32_t idx_off[kN];   // byte offset into the index tile
  uint32_t w_off[kN];     // byte offset of row r in the FP4 tile
  uint32_t sw[kN];        // (2q) ^ (r % 8): swizzled position of the first chunk
  uint32_t lut_off[kN];   // byte offset of this lane's codebook copy (codebook 0 or 1)
  __device__ __forceinline__ void init(int dt, int cb_split) {
#pragma unroll
    for (int it = 0; it < kN; ++it) {
      const int item = it * NT + dt;
      const int r = item & 127, q = item >> 7;
      idx_off[it] = q * 2048 + r * 16;
      w_off[it] = r * 128;
      sw[it] = static_cast<uint32_t>((2 * q) ^ (r & 7));
      lut_off[it] = ((cb_split && q >= 2) ? kLutBytes : 0) + (dt & 31) * 4;
    }
  }
};

template <int NT>
__device__ __forceinline__ void decode_w_tile(const uint8_t* __restrict__ idx, uint32_t lut_s,
                                              uint8_t* __restrict__ wt, const ItemMap<NT>& im) {
#pragma unroll
  for (int it = 0; it < ItemMap<NT>::kN; ++it) {
    const uint4 iv = *reinterpret_cast<const uint4*>(idx + im.idx_off[it]);
    const uint32_t base = lut_s + im.lut_off[it];
    const uint4 o0 = make_uint4(lut16_pair(base, iv.x, 0), lut16_pair(base, iv.x, 2), lut16_pair(base, iv.y, 0),
                                lut16_pair(base, iv.y, 2));
    const uint4 o1 = make_uint4(lut16_pair(base, iv.z, 0), lut16_pair(base, iv.z, 2), lut16_pair(base, iv.w, 0),
                                lut16_pair(base, iv.w, 2));
    *reinterpret_cast<uint4*>(wt + im.w_off[it] + (im.sw[it] << 4)) = o0;
    *reinterpret_cast<uint4*>(wt + im.w_off[it] + ((im.sw[it] ^ 1u) << 4)) = o1;
  }
}

// PreScale+ (Table 4 caption: Ks = 256 entries, ds = 8; Figure 3 b, c: larger ds
// compress the scales further): one scale-codebook index per group of ds
// consecutive block scales of a row.  The packed indices of a 128-row band come in
// units: one 256-channel stage with G = 256/(ds*B) groups per row when ds*B <= 256,
// else one group (G = 1) spanning spu = ds*B/256 stages.
struct SvqGeom {
  // ds in {8, 16, 32}, B in {16, 32}: every quantity below is a power of two, kept
  // with its base-2 logarithm so that the scale decode divides by shifting
  int ds, G, spu, U, lds, lspu;
  __device__ __forceinline__ SvqGeom(int ds_, int B, int KS) {   // ds_ <= 0 (no scale VQ): the default 8
    ds = ds_ > 0 ? ds_ : 8;
    G = max(1, kStageK / (ds * B));
    spu = max(1, ds * B / kStageK);
    lds = 31 - __clz(ds);
    lspu = 31 - __clz(spu);
    U = KS >> lspu;
  }
  // the unit of the band's indices that holds stage ks: [128][G] bytes
  __device__ __forceinline__ const uint8_t* unit(const uint8_t* sidx, int band, int ks) const {
    return sidx + (static_cast<size_t>(band) * U + (ks >> lspu)) * 128 * G;
  }
  // first block of stage ks within its unit
  __device__ __forceinline__ int kb_base(int ks, int B) const { return (ks & (spu - 1)) * (kStageK / B); }
};

// The 32-bit word of block scales kb..kb+3 (kb a multiple of 4, counted from the
// unit's first block) of one row: word (kb mod ds)/4 of the entry that the row's
// index for group kb/ds selects (lds = log2 ds).  Generic loads: the indices and the
// table may sit in shared or global memory.
__device__ __forceinline__ uint32_t svq_word(const uint8_t* row_idx, const uint32_t* scb32, int lds, int kb) {
  return scb32[(static_cast<uint32_t>(row_idx[kb >> lds]) << (lds - 2)) + ((kb & ((1 << lds) - 1)) >> 2)];
}

// A stage's weight scale atoms (A atoms of 128 rows x 4 blocks, the tcgen05 scale
// layout) from the unit's indices; kb0 = the stage's first block within the unit.
template <int A, int NT>
__device__ __forceinline__ void decode_sf_tile(const uint8_t* sidx, int G, const uint32_t* scb32, int lds, int kb0,
                                               uint8_t* __restrict__ sfw, int dt) {
  for (int u = dt; u < 128 * A; u += NT) {   // consecutive threads: consecutive atom words
    const int word = u & 127, a = u >> 7;
    const int r = (word >> 2) + 32 * (word & 3);
    reinterpret_cast<uint32_t*>(sfw + a * 512)[word] = svq_word(sidx + r * G, scb32, lds, kb0 + 4 * a);
  }
}

// PostScale-QB: every block of a QBlock has the QBlock's scale, so the stage's A
// scale atoms are that byte everywhere -- b0 for all of them, or b0 for the first
// half of the stage and b1 for the second when the QBlock is 128 wide along K.
template <int A, int NT>
__device__ __forceinline__ void fill_sf_qbs(uint8_t* __restrict__ sfw, uint32_t b0, uint32_t b1, int dt) {
  const uint32_t w0 = b0 * 0x01010101u, w1 = b1 * 0x01010101u;
  for (int u = dt; u < A * 32; u += NT) {             // 16 bytes a thread, atom u / 32
    const uint32_t v = (u / 32) < A / 2 ? w0 : w1;
    reinterpret_cast<uint4*>(sfw)[u] = make_uint4(v, v, v, v);
  }
}

// Named barriers in their non-aligned form: threads of a warp may reach them from
// divergent paths.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads, so a
// group can take one uniform decision (e.g. all stop after any of them timed out).
__device__ __forceinline__ bool named_bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pin, pout;\n\t"
      "setp.ne.u32 pin, %1, 0;\n\t"
      "barrier.red.and.pred pout, %2, %3, pin;\n\t"
      "selp.u32 %0, 1, 0, pout;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void store_out(void* y, int64_t ldy, int out_bf16, int64_t m, int64_t n, float v) {
  if (out_bf16) {
    reinterpret_cast<uint16_t*>(y)[m * ldy + n] = f32_to_bf16_rne(v);
  } else {
    reinterpret_cast<float*>(y)[m * ldy + n] = v;
  }
}

// ------------------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------------------
template <int FMT, int WSRC, int T, int NCB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_wq,
                const __grid_constant__ GemmParams<1> p) {
  using L = StageLayout<FMT, WSRC, T, NCB>;
  constexpr int STAGES = L::STAGES;
  constexpr int A = L::kAtoms;
  constexpr int XG = L::kXG;
  constexpr int TCOL = T / kColGroups;               // accumulator columns per epilogue warp

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* dec = full + STAGES;
  uint64_t* empty = dec + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  uint8_t* scb_smem = smem + 2048;
  uint8_t* stages = smem + L::CTRL;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K;
  const int KS = K / kStageK;
  const int KB4 = K / L::kB / 4;      // scale atoms per 128 rows over all of K
  const int splits = p.splits;

  // ---- which tile this CTA owns ----
  const int n_tile = blockIdx.x;
  const ExpertPtrs* wp = &p.w[0];
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * T;
  const int64_t m_end = p.M;
  const int sf_group0 = static_cast<int>(m0 / 128);
  const int split = blockIdx.z;
  const int ks_begin = split * p.ks_per_split;
  const int ks_end = min(KS, ks_begin + p.ks_per_split);
  const int nks = ks_end - ks_begin;
  const int nst = nks;
  // Loop invariants in registers (the asm statements below clobber "memory").
  const uint8_t* const w_idx = wp->idx;
  const uint16_t* const w_cb = wp->cb;
  const uint8_t* const w_sf = wp->sf;
  const uint8_t* const w_sidx = wp->sidx;
  const uint8_t* const w_scb = wp->scb;
  const float w_tscale0 = wp->w_tscale;
  const uint8_t* const a_sf = p.a_sf;
  const int qn = p.qn, qk = p.qk;

  // ---- setup ----
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&dec[s], kDecWarps / dec_groups<T>());
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
    prefetch_tensormap(&tmap_x);
    if constexpr (WSRC == WSRC_NATIVE) prefetch_tensormap(&tmap_wq);
  }
  if (warp == 1) {
    __syncwarp();                                  // tcgen05.alloc is warp-aligned
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  // PreScale+: the scale codebook (256 x ds bytes) in shared memory when it is the
  // 2 KB of ds = 8, else read in place (through L1)
  const SvqGeom sv(wp->ds, L::kB, KS);
  const int sv_lds = sv.lds;
  const uint32_t* const scb32 = sv.ds == 8 ? reinterpret_cast<const uint32_t*>(scb_smem)
                                           : reinterpret_cast<const uint32_t*>(w_scb);
  if constexpr (L::kSVQ) {
    if (sv.ds == 8)
      for (int i = threadIdx.x; i < 512; i += kThreads)
        reinterpret_cast<uint32_t*>(scb_smem)[i] = __ldg(reinterpret_cast<const uint32_t*>(w_scb) + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // epilogue state (warps 2..9), kept in registers across the cluster barrier
  uint32_t acc_regs[T <= 32 ? TCOL : 1];
  bool ep_ok = false;
  const int qd = warp & 3;                           // TMEM lane quadrant this warp may read
  const int chalf = (warp - 2) >> 2;                 // which column group of the accumulator
  const int row = qd * 32 + lane;
  const int64_t n = static_cast<int64_t>(n_tile) * 128 + row;
  const int64_t mbase = m0 + chalf * TCOL;           // first token of this warp's columns
  float scale = 1.0f;

  if (warp == 0) {
    // =============================== loader ===============================
    const int cb_per_row = K / qk;
    constexpr bool cb_split = NCB == 2;
    // Token scale groups that exist: the SF buffer holds ceil(M/128) groups of 128
    // rows (dense) -- a 256-token tile at the end of M may cover only one.
    const int groups = static_cast<int>((static_cast<int64_t>(p.M) + 127) / 128);
    const int xg_valid = groups - sf_group0 < XG ? groups - sf_group0 : XG;
    uint32_t tx = T * 128 + xg_valid * A * 512;
    if constexpr (WSRC == WSRC_NATIVE) tx += 16384 + A * 512;
    if constexpr (WSRC == WSRC_VQ_DIRECT) tx += 8192 + (cb_split ? 1024 : 512) + A * 512;
    if constexpr (WSRC == WSRC_VQ_SVQ) tx += 8192 + (cb_split ? 1024 : 512) + 128 * sv.G;
    if constexpr (WSRC == WSRC_VQ_QBS) tx += 8192 + (cb_split ? 1024 : 512);
    const uint8_t* sfx_src = a_sf + static_cast<size_t>(sf_group0) * KB4 * 512;
    const int y0 = static_cast<int>(m0);
    int issued = 0;
    for (int i = 0; i < nst; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1;
      if (i >= STAGES && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1))) break;
      if (elect_one()) {
        const int ks = ks_begin + i;
        const int band = n_tile;
        const int qbn = static_cast<int>((static_cast<int64_t>(band) * 128) / qn);
        const uint8_t* sfw_src = w_sf + static_cast<size_t>(band) * KB4 * 512;
        const uint8_t* idx_src = w_idx + static_cast<size_t>(band) * KS * 8192;
        const uint16_t* cb_src = w_cb + static_cast<size_t>(qbn) * cb_per_row * 256;
        uint8_t* st = stages + s * L::BYTES;
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(st + L::X_OFF, &tmap_x, ks * 128, y0, &full[s]);
#pragma unroll
        for (int g = 0; g < XG; ++g)
          if (g < xg_valid)                          // a missing group's rows are past M: never stored
            bulk_load(st + L::SFX_OFF + g * A * 512, sfx_src + (static_cast<size_t>(g) * KB4 + ks * A) * 512,
                      A * 512, &full[s]);
        if constexpr (WSRC == WSRC_NATIVE) {
          tma_load_2d(st + L::W_OFF, &tmap_wq, ks * 128, n_tile * 128, &full[s]);
          bulk_load(st + L::SFW_OFF, sfw_src + static_cast<size_t>(ks) * A * 512, A * 512, &full[s]);
        } else {
          bulk_load(st + L::IDX_OFF, idx_src + static_cast<size_t>(ks) * 8192, 8192, &full[s]);
          const int qbk = cb_split ? 2 * ks : (ks * kStageK) / qk;
          bulk_load(st + L::CB_OFF, cb_src + static_cast<size_t>(qbk) * 256, cb_split ? 1024 : 512, &full[s]);
          if constexpr (WSRC == WSRC_VQ_DIRECT) {
            bulk_load(st + L::SFW_OFF, sfw_src + static_cast<size_t>(ks) * A * 512, A * 512, &full[s]);
          } else if constexpr (WSRC == WSRC_VQ_SVQ) {
            bulk_load(st + L::SIDX_OFF, sv.unit(w_sidx, band, ks), 128 * sv.G, &full[s]);
          }                                        // PostScale-QB: the decoders write the atoms
        }
      }
      __syncwarp();
      ++issued;
    }
    // Let every copy this warp started land before the CTA can retire.
    for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
      mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    for (int i = 0; i < nst; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) break;
      tc_fence_after();
      const uint8_t* st = stages + s * L::BYTES;
      const uint32_t sfw_s = smem_u32(st + L::SFW_OFF), sfx_s = smem_u32(st + L::SFX_OFF);
      // Scale atoms that arrived by copy go to TMEM while the decoders work.
      if (elect_one()) {
#pragma unroll
        for (int g = 0; g < XG; ++g)
#pragma unroll
          for (int a = 0; a < A; ++a)
            tc_cp_32x128b_warpx4(tmem + L::COL_SFX + (XG == 2 ? 8 * a + 4 * g : 4 * a),
                                 sdesc_sf_atom(sfx_s + (g * A + a) * 512));
        if constexpr (!L::kSfwDec) {
#pragma unroll
          for (int a = 0; a < A; ++a)
            tc_cp_32x128b_warpx4(tmem + L::COL_SFW + 4 * a, sdesc_sf_atom(sfw_s + a * 512));
        }
      }
      __syncwarp();
      if constexpr (L::kVQ) {
        if (!__all_sync(0xffffffffu, mbar_wait(&dec[s], ph))) break;
        tc_fence_after();
      }
      if (elect_one()) {
        if constexpr (L::kSfwDec) {
#pragma unroll
          for (int a = 0; a < A; ++a)
            tc_cp_32x128b_warpx4(tmem + L::COL_SFW + 4 * a, sdesc_sf_atom(sfw_s + a * 512));
        }
        const uint32_t w_s = smem_u32(st + L::W_OFF), x_s = smem_u32(st + L::X_OFF);
        const int il = i;
        const uint32_t d_t = tmem;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t adesc = sdesc_kmajor_sw128(w_s + 32 * j);
          const uint64_t bdesc = sdesc_kmajor_sw128(x_s + 32 * j);
          const uint32_t acc = (il > 0 || j > 0) ? 1u : 0u;
          if constexpr (FMT == FMT_E4M3) {
            constexpr uint32_t idesc = idesc_mxf4(T, 0, 0, 0);
            tc_mma_mxf4nvf4_block16(d_t, adesc, bdesc, idesc, tmem + L::COL_SFW + 4 * j,
                                    tmem + L::COL_SFX + (XG == 2 ? 8 * j : 4 * j), acc);
          } else {
            const int a = j >> 1;
            const uint32_t id = static_cast<uint32_t>(j & 1) * 2;
            const uint32_t idesc = idesc_mxf4(T, 1, static_cast<int>(id), static_cast<int>(id));
            tc_mma_mxf4_block32(d_t, adesc, bdesc, idesc, (tmem + L::COL_SFW + 4 * a) | (id << 30),
                                (tmem + L::COL_SFX + (XG == 2 ? 8 * a : 4 * a)) | (id << 30), acc);
          }
        }
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (elect_one()) tc_commit(accum);
    __syncwarp();
    mbar_wait(accum, 0);      // our own MMAs must finish before the CTA retires
  } else {
    // ======================= decoders, then epilogue ======================
    const int dt = threadIdx.x - 64;
    if constexpr (L::kVQ) {
      // Group g decodes stages g, g + G, ...  One group: codebook copies double-
      // buffered -- stage i decodes through buffer i%2 while the copies of stage
      // i+1 go into the other; one barrier per stage (it also orders stage i's
      // lookups before buffer i%2 is rebuilt).  Two groups: one buffer each, a
      // barrier before and after each rebuild.
      constexpr int G = dec_groups<T>();
      constexpr int GT = kDecThreads / G;            // threads per group
      constexpr int cb_split = NCB == 2;
      constexpr int kBuf = NCB * kLutBytes;
      constexpr int kBufs = 2 / G;                   // copy buffers per group
      const int grp = dt / GT, gt = dt - grp * GT;
      const int bar_id = 2 + grp;
      uint8_t* lut = smem + L::LUT_OFF + grp * kBufs * kBuf;
      const uint32_t lut_s = smem_u32(lut);
      ItemMap<GT> cm;
      cm.init(gt, cb_split);
      auto stage_cb = [&](int i) {
        return reinterpret_cast<const uint16_t*>(stages + (i % STAGES) * L::BYTES + L::CB_OFF);
      };
      bool ok = true;
      int b = 0;
      if (grp < nst) {
        const bool got = mbar_wait(&full[grp % STAGES], (grp / STAGES) & 1);
        if (got) build_lut<GT>(stage_cb(grp), 1 + cb_split, reinterpret_cast<uint32_t*>(lut), gt);
        ok = named_bar_and(bar_id, GT, got);         // one decision for the group
      }
      for (int i = grp; i < nst && ok; i += G) {
        const int s = i % STAGES;
        uint8_t* st = stages + s * L::BYTES;
        uint32_t qs0 = 0, qs1 = 0;                   // PostScale-QB: the stage's QBlock scale(s),
        if constexpr (L::kQBS) {                     // loaded before the decode hides their latency
          const int ks = ks_begin + i;
          const int qbn_w = static_cast<int>((static_cast<int64_t>(n_tile) * 128) / qn);
          const uint8_t* qb = w_sf + static_cast<size_t>(qbn_w) * (K / qk);
          const int qbk = cb_split ? 2 * ks : (ks * kStageK) / qk;
          qs0 = __ldg(qb + qbk);
          qs1 = __ldg(qb + qbk + (cb_split ? 1 : 0));
        }
        decode_w_tile<GT>(st + L::IDX_OFF, lut_s + b * kBuf, st + L::W_OFF, cm);
        if constexpr (L::kSVQ) {
          const int ks = ks_begin + i;
          decode_sf_tile<A, GT>(st + L::SIDX_OFF, sv.G, scb32, sv_lds, sv.kb_base(ks, L::kB), st + L::SFW_OFF, gt);
        }
        if constexpr (L::kQBS) fill_sf_qbs<A, GT>(st + L::SFW_OFF, qs0, qs1, gt);
        fence_proxy_async_smem();                    // each thread's tile writes -> async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&dec[s]);         // one arrival per decoder warp of the group
        const int in = i + G;
        if (in < nst) {                              // this group's next stage
          if (kBufs == 1) named_bar_sync(bar_id, GT);   // lookups of stage i done before the rebuild
          const int nb = kBufs == 2 ? (b ^ 1) : 0;
          const bool got = mbar_wait(&full[in % STAGES], (in / STAGES) & 1);
          if (got) build_lut<GT>(stage_cb(in), 1 + cb_split, reinterpret_cast<uint32_t*>(lut + nb * kBuf), gt);
          ok = named_bar_and(bar_id, GT, got);
          b = nb;
        }
      }
    }
    ep_ok = mbar_wait(accum, 0);
    tc_fence_after();
    float wts = w_tscale0;
    if constexpr (WSRC == WSRC_NATIVE) {
      if (p.w_tscale_dev) wts = *p.w_tscale_dev;
    }
    scale = wts * (p.a_tscale ? *p.a_tscale : 1.0f);
    void* const y = p.y;
    const int64_t ldy = p.ldy;
    const int out_bf16 = p.out_bf16;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(qd * 32) << 16) + chalf * TCOL;
    if constexpr (T <= 32) {
      // this warp's accumulator columns in registers: one TMEM round trip
      __syncwarp();                                  // tcgen05.ld is warp-aligned: converge after the waits
      if constexpr (TCOL == 4) tmem_ld_32x32b_x4(taddr, acc_regs);
      else if constexpr (TCOL == 8) tmem_ld_32x32b_x8(taddr, acc_regs);
      else tmem_ld_32x32b_x16(taddr, acc_regs);
      tmem_ld_wait();
      if (ep_ok) {
        if (splits > 1) {
          const uint32_t rank = cluster_ctarank();
          if (rank != 0) {
            // partial tile -> rank 0's receive slot (rank-1), [T][128] floats
            const uint32_t slot = smem_u32(smem + L::RED_OFF) + (((rank - 1) * T + chalf * TCOL) * 128 + row) * 4;
            const uint32_t remote = mapa_shared(slot, 0);
#pragma unroll
            for (int c = 0; c < TCOL; ++c) st_cluster_f32(remote + c * 128 * 4, __uint_as_float(acc_regs[c]));
          }
        } else {
#pragma unroll
          for (int c = 0; c < TCOL; ++c)
            if (mbase + c < m_end) store_out(y, ldy, out_bf16, mbase + c, n, __uint_as_float(acc_regs[c]) * scale);
        }
      }
    } else {
      // Split-K of a 128-token tile through the workspace: this rank's scaled partial,
      // token-major [T][128] FP32 (a warp's stores are coalesced); the rank of the tile
      // that arrives last at its counter adds the partials in rank order (products and
      // sums rounded separately).
      const size_t tile = static_cast<size_t>(blockIdx.y) * gridDim.x + n_tile;
      float* const part = p.red_part ? p.red_part + tile * splits * (static_cast<size_t>(T) * 128) : nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < TCOL; c0 += 32) {
        uint32_t v[32];
        __syncwarp();                                // tcgen05.ld is warp-aligned
        tmem_ld_32x32b_x32(taddr + c0, v);
        tmem_ld_wait();
        if (!ep_ok) continue;
        if (part) {
          float* const dst =
              part + static_cast<size_t>(split) * (T * 128) + static_cast<size_t>(chalf * TCOL + c0) * 128 + row;
#pragma unroll
          for (int c = 0; c < 32; ++c) __stcg(dst + c * 128, __fmul_rn(__uint_as_float(v[c]), scale));
          continue;
        }
        const int64_t rem = m_end - (mbase + c0);
        if (rem <= 0) continue;
        const int cmax = rem < 32 ? static_cast<int>(rem) : 32;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < cmax) store_out(y, ldy, out_bf16, mbase + c0 + c, n, __uint_as_float(v[c]) * scale);
      }
      if (part) {
        __threadfence();                             // the partial is visible before the ticket
        named_bar_sync(4, kDecThreads);
        uint32_t* const last = tmem_slot + 1;
        if (threadIdx.x == 64)                       // every rank arrives once, also after a failed wait
          *last = atomicInc(p.red_ctr + tile, static_cast<unsigned>(splits - 1)) == static_cast<unsigned>(splits - 1);
        named_bar_sync(4, kDecThreads);
        if (*last) {
          __threadfence();                           // the other ranks' partials are visible
          const float* const src = part + static_cast<size_t>(chalf * TCOL) * 128 + row;
#pragma unroll 1
          for (int c0 = 0; c0 < TCOL; c0 += 32) {
            // one rank's 32 values at a time, all loads in flight together
            float sum[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) sum[c] = __ldcg(src + (c0 + c) * 128);
            for (int r = 1; r < splits; ++r) {
              float t[32];
#pragma unroll
              for (int c = 0; c < 32; ++c) t[c] = __ldcg(src + static_cast<size_t>(r) * (T * 128) + (c0 + c) * 128);
#pragma unroll
              for (int c = 0; c < 32; ++c) sum[c] = __fadd_rn(sum[c], t[c]);
            }
            if (!ep_ok) continue;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (mbase + c0 + c < m_end) store_out(y, ldy, out_bf16, mbase + c0 + c, n, sum[c]);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
  if constexpr (T <= 32) {
    if (splits > 1) {
      // All partial tiles have landed in rank 0's shared memory after this barrier.
      __syncwarp();
      cluster_sync_all();
      if (warp >= 2 && ep_ok && cluster_ctarank() == 0) {
        const float* red = reinterpret_cast<const float*>(smem + L::RED_OFF);
#pragma unroll
        for (int c = 0; c < TCOL; ++c) {
          float sum = __uint_as_float(acc_regs[c]);
          for (int r = 1; r < splits; ++r) sum += red[((r - 1) * T + chalf * TCOL + c) * 128 + row];
          if (mbase + c < m_end) store_out(p.y, p.ldy, p.out_bf16, mbase + c, n, sum * scale);
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------
// Decode dump for small QBlocks (64 rows or 64 input channels, down to 64 x 64: the fine
// end of Figure 3's QBlock sweep).  A 128 x 256 tile-stage then draws on up to 8
// codebooks ([2 row halves][4 K-quarters]), too many for per-lane codebook copies, so
// the stage's codebooks sit once in shared memory and every index is looked up
// directly (bank conflicts allowed).  Writes the same plain layouts as the decode
// pass: FP4 codes [N, ldq], SF-layout scales.  Grid (N/128, K/256).
// ------------------------------------------------------------------------------------
template <int FMT, int WSRC>
__global__ void __launch_bounds__(128)
    decode_dump_small_kernel(const ExpertPtrs w, int N, int K, int qn, int qk, uint8_t* __restrict__ q_out,
                             int64_t ldq, uint8_t* __restrict__ sf_out) {
  constexpr int B = FMT == FMT_E8M0 ? 32 : 16;
  constexpr int A = kStageK / B / 4;                   // scale atoms per 128 rows per stage
  __shared__ uint16_t cbs[8 * 256];
  const int n_tile = blockIdx.x, ks = blockIdx.y, KS = K / kStageK;
  const int rows_cb = qn < kTileN ? kTileN / qn : 1;   // codebook rows in the 128-row tile
  const int qke = qk < kStageK ? qk : kStageK;
  const int nkq = kStageK / qke;                       // codebooks along K in the stage
  const int qbn0 = static_cast<int>((static_cast<int64_t>(n_tile) * kTileN) / qn);
  const int qbk0 = static_cast<int>((static_cast<int64_t>(ks) * kStageK) / qk);
  // the stage's codebooks, [rows_cb][nkq][256] entries (at most 8 x 512 bytes)
  for (int i = threadIdx.x; i < rows_cb * nkq * 128; i += 128) {
    const int c = i >> 7, wd = i & 127, rh = c / nkq, kq = c % nkq;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(
        w.cb + (static_cast<size_t>(qbn0 + rh) * (K / qk) + qbk0 + kq) * 256);
    reinterpret_cast<uint32_t*>(cbs)[i] = __ldg(src + wd);
  }
  __syncthreads();
  // item (r, q): the 16 indices of row r in K-quarter q -> 32 bytes of FP4 codes
  const uint8_t* tile = w.idx + (static_cast<size_t>(n_tile) * KS + ks) * 8192;
  for (int it = threadIdx.x; it < 512; it += 128) {
    const int r = it & 127, q = it >> 7;
    const uint16_t* cb = cbs + ((r / (kTileN / rows_cb)) * nkq + (q * 64) / qke) * 256;
    const uint4 iv = ldg_nc_v4(tile + q * 2048 + r * 16);
    const uint32_t x[4] = {iv.x, iv.y, iv.z, iv.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t b = x[j >> 1] >> (16 * (j & 1));
      o[j] = static_cast<uint32_t>(cb[b & 0xFF]) | (static_cast<uint32_t>(cb[(b >> 8) & 0xFF]) << 16);
    }
    uint8_t* dst = q_out + (static_cast<int64_t>(n_tile) * kTileN + r) * ldq + static_cast<int64_t>(ks) * 128 + q * 32;
    *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + 16) = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // the tile-stage's scale atoms in the SF layout
  const size_t wsf = (static_cast<size_t>(n_tile) * (K / B / 4) + static_cast<size_t>(ks) * A) * 512;
  if constexpr (WSRC == WSRC_VQ_DIRECT) {
    for (int i = threadIdx.x; i < A * 32; i += 128)
      reinterpret_cast<uint4*>(sf_out + wsf)[i] = ldg_nc_v4(w.sf + wsf + static_cast<size_t>(i) * 16);
  } else if constexpr (WSRC == WSRC_VQ_SVQ) {
    const SvqGeom sv(w.ds, B, KS);
    decode_sf_tile<A, 128>(sv.unit(w.sidx, n_tile, ks), sv.G, reinterpret_cast<const uint32_t*>(w.scb), sv.lds,
                           sv.kb_base(ks, B), sf_out + wsf, threadIdx.x);
  } else {
    // PostScale-QB: word (r % 32) * 4 + g of atom a holds the scales of rows 32 g + r % 32
    // (one QBlock row: qn >= 64) for blocks 4a..4a+3, each from its QBlock
    for (int i = threadIdx.x; i < A * 128; i += 128) {
      const int a = i >> 7, g = i & 3;
      const int qbn = static_cast<int>((static_cast<int64_t>(n_tile) * kTileN + 32 * g) / qn);
      uint32_t v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int64_t c = static_cast<int64_t>(ks) * kStageK + static_cast<int64_t>(4 * a + b) * B;
        v |= static_cast<uint32_t>(__ldg(w.sf + static_cast<size_t>(qbn) * (K / qk) + c / qk)) << (8 * b);
      }
      reinterpret_cast<uint32_t*>(sf_out + wsf)[i] = v;
    }
  }
}

}  // namespace mxc
