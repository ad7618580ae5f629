// decode_pass.cuh -- decode once: a VQ weight into MX-native FP4 codes [N, K/2] and
// SF-layout scales, the operands of the native block-scaled GEMM (the decode-once
// prefill path) and the output of mxc_decode_weight.
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale", abstract: the VQ
// storage is turned into MX-native FP4 operands, never into a high-precision weight.
// One CTA takes 128 weight rows x 8 stages of 256 input channels (grid (N/128,
// ceil(K/2048))) and decodes them the way the decode GEMV does:
//   * the loader requests the stages' codebooks, index quarters 0 and 1 into shared
//     memory and quarters 2 and 3 into L2, then copies quarters 2 and 3 into the
//     quarter buffers as quarters 0 and 1 are decoded;
//   * decoder lane l lays out the codebook of stage l mod 8 in its own bank (32
//     per-lane copies, one entry per 32-bit word) once, and the 16 decoder warps
//     decode K-quarter by K-quarter into 128-byte-swizzled stage tiles -- the codebook
//     copies serve all 8 stages, instead of being laid out again for every stage;
//   * one 3-D tensor store writes the 8 tiles into the FP4 matrix (the tiles' swizzle
//     is the store map's), and the decoder threads write the stages' scale atoms to
//     the SF layout: copied (direct scales), built from the scale indices (PreScale+)
//     or filled with the QBlock's byte (PostScale-QB).
// Nothing here waits on another CTA; every copy and store lands before the CTA retires.
#pragma once

#include "pair_kernel.cuh"

namespace mxc {

constexpr int kPassThreads = 32 + kDecThreads;   // loader warp + 16 decoder warps

template <int FMT, int WSRC>
struct PassLayout {
  static constexpr int kB = FMT == FMT_E8M0 ? 32 : 16;
  static constexpr int A = kStageK / kB / 4;            // scale atoms per 128 rows per stage
  static constexpr int S = kGemvMaxStages;
  static constexpr int W_OFF = 0;                       // S x [128][128 B] decoded tiles, 128-byte swizzle
  static constexpr int IDX_OFF = W_OFF + S * 16384;     // 2 quarter buffers x [S][128][16 B]
  static constexpr int IDX_BUF = S * 2048;
  static constexpr int LUT_OFF = IDX_OFF + 2 * IDX_BUF; // 256 words x 32 lanes
  // the stages' codebooks (at most 16 x 512 B) land in the second half of the last
  // stage's tile, which is not written before the codebook copies are laid out
  static constexpr int CB_OFF = W_OFF + (S - 1) * 16384 + 8192;
  static constexpr int CTRL_OFF = LUT_OFF + kGemvLutBytes;
  static constexpr int SMEM = 1024 + CTRL_OFF + 128;
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int x, int y, int z, const void* src) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(smem_u32(src))
               : "memory");
}

template <int FMT, int WSRC>
__global__ void __launch_bounds__(kPassThreads, 1)
    decode_pass_kernel(const __grid_constant__ CUtensorMap tmap_idx, const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ ExpertPtrs w, int N, int K, int qn, int qk, int box,
                       uint8_t* __restrict__ sf_out) {
  using L = PassLayout<FMT, WSRC>;
  constexpr int A = L::A;
  constexpr bool kSVQ = WSRC == WSRC_VQ_SVQ;
  constexpr bool kQBS = WSRC == WSRC_VQ_QBS;
  static_assert(kDecWarps == 16, "decode map assumes 16 decoder warps");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::CTRL_OFF);
  uint64_t* full = bars;            // [4] K-quarter j of the stages' index slabs
  uint64_t* dec_ph = bars + 4;      // [4] K-quarter j decoded (one arrival per decoder warp)
  uint64_t* bar_cb = bars + 8;      // the stages' codebooks

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = K / kStageK, KB4 = K / L::kB / 4;
  const int n_tile = blockIdx.x, ks0 = blockIdx.y * L::S;
  const int rn = min(L::S, KS - ks0);                   // this CTA's stages
  const int H = qk == 128 ? 2 : 1;                      // codebooks per stage along K
  const int qbn = static_cast<int>((static_cast<int64_t>(n_tile) * 128) / qn);
  const uint8_t* const w_idx = w.idx + (static_cast<size_t>(n_tile) * KS + ks0) * 8192;
  const uint16_t* const w_cb = w.cb + static_cast<size_t>(qbn) * (K / qk) * 256;
  const int qa = H == 2 ? 2 * ks0 : (ks0 * kStageK) / qk;   // the stages' codebooks [qa, qz]
  const int qz = H == 2 ? 2 * (ks0 + rn) - 1 : ((ks0 + rn - 1) * kStageK) / qk;

  if (warp == 0) {
    if (lane < 9) mbar_init(bars + lane, (lane >= 4 && lane < 8) ? kDecWarps : 1);
    __syncwarp();
    if (lane == 0) {
      fence_mbar_init();
      prefetch_tensormap(&tmap_idx);
      prefetch_tensormap(&tmap_q);
      const uint32_t cb_bytes = static_cast<uint32_t>(qz - qa + 1) * 512;
      mbar_arrive_expect_tx(bar_cb, cb_bytes);
      bulk_load(smem + L::CB_OFF, w_cb + static_cast<size_t>(qa) * 256, cb_bytes, bar_cb);
      // quarter j of the stages: box {2048 B, 1, box stages, 1}; stages past K arrive
      // zero-filled and are not used
      for (int j = 0; j < 2; ++j) {
        mbar_arrive_expect_tx(&full[j], box * 2048);
        tma_load_4d(smem + L::IDX_OFF + j * L::IDX_BUF, &tmap_idx, 0, j, ks0, n_tile, &full[j]);
      }
      for (int s = 0; s < rn; ++s) l2_prefetch_bulk(w_idx + static_cast<size_t>(s) * 8192 + 4096, 4096);
    }
  }
  __syncthreads();

  if (warp == 0) {
    // =============================== loader ===============================
    int issued_q = 2;
    if (elect_one()) {
      for (int j = 2; j < 4; ++j) {                    // K-quarter j of every stage (from L2 by now)
        if (!mbar_wait(&dec_ph[j - 2], 0)) break;      // its buffer has been decoded
        mbar_arrive_expect_tx(&full[j], box * 2048);
        tma_load_4d(smem + L::IDX_OFF + (j % 2) * L::IDX_BUF, &tmap_idx, 0, j, ks0, n_tile, &full[j]);
        issued_q = j + 1;
      }
    }
    issued_q = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(issued_q)));
    if (lane == 0) {                                   // every copy lands before the CTA retires
      mbar_wait(bar_cb, 0);
      for (int j = 0; j < issued_q; ++j) mbar_wait(&full[j], 0);
    }
    __syncwarp();
    return;
  }

  // ================================ decoders ================================
  const int dw = warp - 1, dt = threadIdx.x - 32;      // decoder warp 0..15, thread 0..511
  const int s_l = lane & 7;                            // this lane's stage
  const int q = dw * 4 + (lane >> 3);                  // 64 threads per stage
  const bool active = s_l < rn;
  // entries [16 kb, 16 kb + 16) of the codebook of this lane's stage; over the 16 warps
  // each lane covers all 256 entries, and the 8 lanes of a quarter warp read 8
  // different bank groups (the two 16-byte halves in an order alternating with the stage)
  const int kb = (dw + (s_l >> 1)) & 15;
  const int h0 = s_l & 1;
  auto cb_words = [&](int epoch, uint4* c0, uint4* c1) {
    const int ks = ks0 + s_l;
    const int qbk = H == 2 ? 2 * ks + epoch : (ks * kStageK) / qk;
    const uint8_t* cp = smem + L::CB_OFF + (qbk - qa) * 512 + 32 * kb;
    const uint4 first = *reinterpret_cast<const uint4*>(cp + 16 * h0);
    const uint4 second = *reinterpret_cast<const uint4*>(cp + 16 * (1 - h0));
    *c0 = h0 ? second : first;
    *c1 = h0 ? first : second;
  };
  uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0, d0 = c0, d1 = c0;
  const bool cb_ok = mbar_wait(bar_cb, 0);
  if (active && cb_ok) {                               // into registers: the staging is overwritten
    cb_words(0, &c0, &c1);
    if (H == 2) cb_words(1, &d0, &d1);
  }
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L::LUT_OFF) + (16 * kb) * 32 + lane;
  auto lay_out = [&](const uint4& a, const uint4& b) {
    if (!active) return;
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lut[(2 * i) * 32] = v[i] & 0xFFFFu;
      lut[(2 * i + 1) * 32] = v[i] >> 16;
    }
  };
  lay_out(c0, c1);
  named_bar_sync(2, kDecThreads);                      // all copies written
  const uint32_t lut_lane = smem_u32(smem + L::LUT_OFF) + lane * 4;
  const uint8_t* idx_l = smem + L::IDX_OFF + s_l * 2048;
  uint8_t* wt = smem + L::W_OFF + s_l * 16384;
  bool ok = cb_ok;
  for (int j = 0; j < 4; ++j) {
    if (H == 2 && j == 2) {                            // second half of each stage: its own codebook
      named_bar_sync(2, kDecThreads);
      lay_out(d0, d1);
      named_bar_sync(2, kDecThreads);
    }
    const bool landed = mbar_wait(&full[j], 0);
    ok = ok && landed;
    if (active && landed) decode_quarter_rows(lut_lane, idx_l + (j % 2) * L::IDX_BUF, wt, q, s_l, j);
    __syncwarp();
    if (lane == 0) mbar_arrive(&dec_ph[j]);
  }
  fence_proxy_async_smem();                            // tile writes -> the tensor store's reads
  named_bar_sync(2, kDecThreads);                      // all tiles complete
  if (dt == 0 && ok) {
    tma_store_3d(&tmap_q, 0, n_tile * 128, ks0, smem + L::W_OFF);
    bulk_commit_group();
  }
  // the stages' scale atoms, SF layout: A atoms of 512 bytes per stage, contiguous
  uint8_t* const sfo = sf_out + (static_cast<size_t>(n_tile) * KB4 + static_cast<size_t>(ks0) * A) * 512;
  if constexpr (kSVQ) {
    // groups of 128 threads, stage s = group, group + 4
    const SvqGeom sv(w.ds, L::kB, KS);
    const uint32_t* scb32 = reinterpret_cast<const uint32_t*>(w.scb);
    for (int s = dt >> 7; s < rn; s += 4)
      decode_sf_tile<A, 128>(sv.unit(w.sidx, n_tile, ks0 + s), sv.G, scb32, sv.lds, sv.kb_base(ks0 + s, L::kB),
                             sfo + s * A * 512, dt & 127);
  } else if constexpr (kQBS) {
    const uint8_t* qbrow = w.sf + static_cast<size_t>(qbn) * (K / qk);
    for (int s = dt >> 7; s < rn; s += 4) {
      const int ks = ks0 + s;
      const int qbk = H == 2 ? 2 * ks : (ks * kStageK) / qk;
      fill_sf_qbs<A, 128>(sfo + s * A * 512, __ldg(qbrow + qbk), __ldg(qbrow + qbk + (H == 2 ? 1 : 0)), dt & 127);
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(w.sf + (static_cast<size_t>(n_tile) * KB4 +
                                                              static_cast<size_t>(ks0) * A) * 512);
    for (int i = dt; i < rn * A * 32; i += kDecThreads) reinterpret_cast<uint4*>(sfo)[i] = __ldg(src + i);
  }
  if (dt == 0) bulk_wait_group_read0();                // the store has read the tiles
}

}  // namespace mxc
