// act_quant.cu -- BF16 -> MX FP4 activation quantization (W4A4 activations).
//
// "MXCode: Vector Quantization for MX-Native Inference at Scale": W4A4 on native
// block-scaled FP4 (abstract; Table 2 caption), formats E8M0-B32 and E4M3-B16
// with an FP32 tensor scale (Table 1).  The pages give no activation recipe;
// this follows the OCP MX rule (block scale from the block amax, E2M1 round to
// nearest even, saturate at +-6) with the E4M3 tensor scale amax/(6*448).
//
// One thread quantizes one block (32 or 16 elements): vector loads of BF16,
// block amax, scale byte, 32/16 E2M1 codes decided by the sign of an exact
// fused multiply-add against each rounding midpoint, one vector store of FP4.
// The work is HBM-bound (read 2 bytes/element, write ~0.53).
#pragma once

#include <cstdint>

#include "mxc_device.cuh"
#include "mxc_internal.h"

namespace mxc {

// Byte offset of scale (r, kb) in the SF layout (see mxc.h).
__device__ __forceinline__ size_t sf_offset(int64_t r, int kb, int kb_per_row) {
  return (static_cast<size_t>(r >> 7) * (kb_per_row >> 2) + (kb >> 2)) * 512 + (r & 31) * 16 +
         ((r >> 5) & 3) * 4 + (kb & 3);
}

// E4M3 (no infinities, max 448) of a non-negative float: round to nearest,
// ties to even mantissa, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode_satfinite(float v) {
  if (!(v < 448.0f)) return 0x7E;                        // >= 448 (and +inf)
  if (v < 0.015625f) {                                   // below 2^-6: subnormal grid m * 2^-9
    return static_cast<uint32_t>(__float2int_rn(v * 512.0f));   // exact scaling, RNE; 8 -> 0x08
  }
  const uint32_t u = __float_as_uint(v);
  uint32_t x = u >> 20;                                  // exponent + top 3 mantissa bits
  const uint32_t rem = u & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (x & 1u))) x += 1;
  const uint32_t b = x - ((127u - 7u) << 3);             // rebias 127 -> 7
  return b > 0x7Eu ? 0x7Eu : b;
}

__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xF, m = b & 7;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// 2^e for e in [-127, 127] as an exact float (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// E2M1 code of x / d, round half to even, saturating at 6, sign of x kept.
// Each midpoint test uses the sign of fma(mu, d, -|x|), which is the sign of
// the exact value mu*d - |x| (one rounding never flips a sign).  The code is
// the number of midpoints |x|/d lies above, found by a three-level binary
// search: 1.75 first (tie -> 2.0, code 4), then 3.5 or 0.75 (ties -> 4.0 /
// 1.0, the even codes above), then 5, 2.5, 1.25 or 0.25 (ties -> 4.0, 2.0, 1.0,
// 0: the even codes below).
__device__ __forceinline__ uint32_t e2m1_code(float x, float d) {
  const float a = fabsf(x);
  const bool hi = __fmaf_rn(1.75f, d, -a) <= 0.0f;                // a >= 1.75 d
  const bool mid = __fmaf_rn(hi ? 3.5f : 0.75f, d, -a) <= 0.0f;   // a >= 3.5 d / 0.75 d
  const float mu = hi ? (mid ? 5.0f : 2.5f) : (mid ? 1.25f : 0.25f);
  const bool lo = __fmaf_rn(mu, d, -a) < 0.0f;                     // a > mu d
  const uint32_t c = (hi ? 4u : 0u) + (mid ? 2u : 0u) + (lo ? 1u : 0u);
  return c | ((__float_as_uint(x) >> 28) & 8u);
}

// E2M1 codes of two FP32 values by the hardware format conversion: round to nearest,
// ties to even, saturating at +-6, the sign kept (also on zero); hi in bits 4..7, lo in
// bits 0..3.  With an E8M0 block scale d = 2^e, x / d = x * 2^-e is exact (a result
// below the normal range is far below the first midpoint 0.25 and codes 0 either
// way), so these are exactly the codes e2m1_code(x, d) decides -- for every BF16 x
// and every e in [-127, 127], checked exhaustively on the GPU against e2m1_code.
__device__ __forceinline__ uint32_t e2m1x2_rn(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t.reg .b16 h;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "mov.b16 h, {t, 0};\n\tcvt.u32.u16 %0, h;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------------------------
// SwiGLU of the MoE projections, one FP32 operation per step (so that the codes of
// its quantization are decided in exactly this arithmetic).  E(x) = e^x by Cody and
// Waite's reduction x = n ln2 + r (ln2 split into a 9-bit head, so n * head is
// exact, and the rest), the degree-7 Taylor polynomial of e^r by Horner's rule and
// the exact scaling by 2^n; +inf above 88 and 0 below -86.  No fused multiply-add.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ float exp_fp32(float x) {
  const float n = rintf(__fmul_rn(x, 1.44269504088896341f));
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(n, 0.693359375f)),
                            __fmul_rn(n, static_cast<float>(0.6931471805599453 - 0.693359375)));
  float q = static_cast<float>(1.0 / 5040.0);
  q = __fadd_rn(__fmul_rn(q, r), static_cast<float>(1.0 / 720.0));
  q = __fadd_rn(__fmul_rn(q, r), static_cast<float>(1.0 / 120.0));
  q = __fadd_rn(__fmul_rn(q, r), static_cast<float>(1.0 / 24.0));
  q = __fadd_rn(__fmul_rn(q, r), static_cast<float>(1.0 / 6.0));
  q = __fadd_rn(__fmul_rn(q, r), 0.5f);
  q = __fadd_rn(__fmul_rn(q, r), 1.0f);
  q = __fadd_rn(__fmul_rn(q, r), 1.0f);
  const int ni = min(127, max(-126, static_cast<int>(n)));
  const float e = __fmul_rn(q, __int_as_float((ni + 127) << 23));
  return x > 88.0f ? __int_as_float(0x7F800000) : x < -86.0f ? 0.0f : e;
}

// h = (g / (1 + E(-g))) * u
__device__ __forceinline__ float swiglu_fp32(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, exp_fp32(-g))), u);
}

// MX quantization of one block of B FP32 values (B = 32: E8M0 scale; B = 16: E4M3
// scale over the given tensor scale s), the rule of quantize_block applied to FP32
// instead of BF16 input: q receives the B/8 words of packed E2M1 codes (element 2i
// in the low nibble of byte i), sfb the scale byte.
template <int B>
__device__ __forceinline__ void quantize_block_f32(const float (&v)[B], bool e4m3, float s, uint32_t (&q)[B / 8],
                                                   uint32_t& sfb) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < B; ++i) a = fmaxf(a, fabsf(v[i]));
  float d = 0.0f;
  if (!e4m3) {
    const uint32_t u = __float_as_uint(a);
    if (a == 0.0f) {
      sfb = 0;
    } else {
      const uint32_t E = (u >> 23) & 0xFF;
      const int flog = E ? static_cast<int>(E) - 127 : (31 - __clz(u & 0x7FFFFF)) - 149;
      const int e = min(127, max(-127, flog - 2));
      sfb = static_cast<uint32_t>(e + 127);
      // power-of-two scale: the codes of the exact quotients by the format conversion
      const float inv = exp2_int(-e);
#pragma unroll
      for (int i = 0; i < B / 8; ++i) q[i] = 0;
#pragma unroll
      for (int i = 0; i < B / 2; ++i)
        q[i / 4] |= e2m1x2_rn(v[2 * i + 1] * inv, v[2 * i] * inv) << (8 * (i % 4));
      return;
    }
  } else {
    sfb = e4m3_encode_satfinite(__fdiv_rn(__fdiv_rn(a, 6.0f), s));
    d = sfb ? __fmul_rn(e4m3_decode(sfb), s) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < B / 8; ++i) q[i] = 0;
#pragma unroll
  for (int i = 0; i < B; ++i) {
    const uint32_t c = d == 0.0f ? ((__float_as_uint(v[i]) >> 28) & 8u) : e2m1_code(v[i], d);
    q[i / 8] |= c << (4 * (i % 8));
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Quantizes one block of B = 32 or 16 BF16 values held as B/2 packed words.
template <int B>
__device__ __forceinline__ void quantize_block(const uint32_t (&w)[B / 2], bool e4m3, float s,
                                               uint32_t (&q)[B / 8], uint32_t& sf_byte) {
  uint32_t amax_bits = 0;
#pragma unroll
  for (int i = 0; i < B / 2; ++i) {
    amax_bits = max(amax_bits, w[i] & 0x7FFFu);
    amax_bits = max(amax_bits, (w[i] >> 16) & 0x7FFFu);
  }
  const float amax = __uint_as_float(amax_bits << 16);
  float d = 0.0f;
  if (!e4m3) {
    if (amax_bits == 0) {
      sf_byte = 0;
    } else {
      const uint32_t u = amax_bits << 16;
      const uint32_t E = (u >> 23) & 0xFF;
      const int flog = E ? static_cast<int>(E) - 127 : (31 - __clz(u & 0x7FFFFF)) - 149;
      const int e = min(127, max(-127, flog - 2));
      sf_byte = static_cast<uint32_t>(e + 127);
      // power-of-two scale: the codes of the exact quotients by the format conversion
      const float inv = exp2_int(-e);
#pragma unroll
      for (int i = 0; i < B / 8; ++i) q[i] = 0;
#pragma unroll
      for (int i = 0; i < B / 2; ++i)
        q[i / 4] |= e2m1x2_rn(bf16_hi(w[i]) * inv, bf16_lo(w[i]) * inv) << (8 * (i % 4));
      return;
    }
  } else {
    const float t = __fdiv_rn(__fdiv_rn(amax, 6.0f), s);
    sf_byte = e4m3_encode_satfinite(t);
    d = sf_byte ? __fmul_rn(e4m3_decode(sf_byte), s) : 0.0f;
  }
#pragma unroll
  for (int i = 0; i < B / 8; ++i) q[i] = 0;
#pragma unroll
  for (int i = 0; i < B / 2; ++i) {
    const float x0 = bf16_lo(w[i]), x1 = bf16_hi(w[i]);
    uint32_t c0, c1;
    if (d == 0.0f) {  // all-zero block, or an E4M3 scale that rounded to 0: signed zeros
      c0 = (w[i] >> 12) & 8u;
      c1 = (w[i] >> 28) & 8u;
    } else {
      c0 = e2m1_code(x0, d);
      c1 = e2m1_code(x1, d);
    }
    q[i / 4] |= (c0 | (c1 << 4)) << (8 * (i % 4));
  }
}

// ------------------------------------------------------------------------------------
// Tensor amax (E4M3 path): max |x| over [M, K], as FP32 bits, via atomicMax on a
// zero-initialised word (max is order independent, so the result is deterministic).
// ------------------------------------------------------------------------------------
__global__ void amax_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                            unsigned int* __restrict__ amax_out) {
  const uint32_t chunks_per_row = static_cast<uint32_t>(K / 8);
  const uint32_t total = static_cast<uint32_t>(M) * chunks_per_row;
  uint32_t m = 0;
  for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < total; c += gridDim.x * blockDim.x) {
    const uint32_t r = c / chunks_per_row, k8 = c - r * chunks_per_row;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + k8 * 8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m = max(m, w[i] & 0x7FFFu);
      m = max(m, (w[i] >> 16) & 0x7FFFu);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(amax_out, m << 16);
}

// One (scale row, block) unit: dense mode maps scale row = data row (rows past M
// only get zero scales); grouped mode maps padded scale rows back to data rows
// (offsets and tile_prefix: the CTA's shared-memory copies).
template <int B>
__device__ __forceinline__ void quantize_unit(const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                              int e4m3, float s, uint8_t* __restrict__ q, int64_t ldq,
                                              uint8_t* __restrict__ sf, uint32_t u, int kb_per_row,
                                              const int32_t* __restrict__ offsets,
                                              const int32_t* __restrict__ tile_prefix, int32_t n_groups) {
  const uint32_t pr32 = u / static_cast<uint32_t>(kb_per_row);
  const int64_t pr = pr32;                    // scale row
  const int kb = static_cast<int>(u - pr32 * static_cast<uint32_t>(kb_per_row));
  int64_t r = pr;                             // data row, -1 = padding
  if (tile_prefix) {
    int lo = 0, hi = n_groups - 1;            // group g with tile_prefix[g]*128 <= pr
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<int64_t>(tile_prefix[mid]) * 128 <= pr) lo = mid; else hi = mid - 1;
    }
    const int64_t local = pr - static_cast<int64_t>(tile_prefix[lo]) * 128;
    r = local < offsets[lo + 1] - offsets[lo] ? offsets[lo] + local : -1;
  } else if (pr >= M) {
    r = -1;
  }
  uint32_t sfb = 0;
  if (r >= 0) {
    const uint16_t* src = x + r * ldx + static_cast<int64_t>(kb) * B;
    uint32_t w[B / 2];
#pragma unroll
    for (int i = 0; i < B / 8; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
    uint32_t qw[B / 8];
    quantize_block<B>(w, e4m3 != 0, s, qw, sfb);
    uint8_t* dst = q + r * ldq + static_cast<int64_t>(kb) * (B / 2);
    if (B == 32) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(qw[0], qw[1], qw[2], qw[3]);
    } else {
      *reinterpret_cast<uint2*>(dst) = make_uint2(qw[0], qw[1]);
    }
  }
  sf[sf_offset(pr, kb, kb_per_row)] = static_cast<uint8_t>(sfb);
}

// ------------------------------------------------------------------------------------
// Quantization.  One thread per (scale row, block).  Dense mode: scale row = data
// row, rows in [M, round_up(M,128)) only get zero scales.  Grouped mode: scale
// rows are padded per group to multiples of 128 (tile_prefix from the group
// prologue) and mapped back to data rows.
// ------------------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(256) quantize_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx, int e4m3,
    const float* __restrict__ tscale_in, const unsigned int* __restrict__ amax_ws,
    uint8_t* __restrict__ q, int64_t ldq, uint8_t* __restrict__ sf, float* __restrict__ tscale_out,
    int64_t sf_rows, const int32_t* __restrict__ offsets, const int32_t* __restrict__ tile_prefix,
    int32_t n_groups) {
  // grouped mode: the group offsets and tile prefix once per CTA into shared memory,
  // so that each unit's group search costs shared-memory loads, not L2 round trips
  __shared__ int32_t off_s[kMaxGroups + 1], tp_s[kMaxGroups + 1];
  if (tile_prefix) {
    for (int g = threadIdx.x; g <= n_groups; g += blockDim.x) {
      off_s[g] = offsets[g];
      tp_s[g] = tile_prefix[g];
    }
    __syncthreads();
    offsets = off_s;
    tile_prefix = tp_s;
  }
  const int kb_per_row = static_cast<int>(K / B);
  float s = 1.0f;
  if (e4m3) {
    if (tscale_in) {
      s = *tscale_in;
    } else {
      const float amax = __uint_as_float(*amax_ws);
      s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
    }
  }
  if (tscale_out && blockIdx.x == 0 && threadIdx.x == 0) *tscale_out = s;
  int64_t rows_total = sf_rows;
  if (tile_prefix) rows_total = min(sf_rows, static_cast<int64_t>(tile_prefix[n_groups]) * 128);
  const uint32_t units = static_cast<uint32_t>(rows_total * kb_per_row);
  for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x)
    quantize_unit<B>(x, M, K, ldx, e4m3, s, q, ldq, sf, u, kb_per_row, offsets, tile_prefix, n_groups);
}

// Small activations (decode batches): one launch of one 16-CTA (else 8-CTA) cluster, one pass.
// Each thread loads its (at most two) blocks into registers once; for E4M3 the CTA
// maxima are pushed into every CTA's shared memory (distributed shared memory,
// one cluster barrier), so each thread then has the tensor amax locally and
// quantizes its blocks from registers (a relaxed cluster arrive at the start and
// its wait before the pushes make sure every CTA runs before it is written to).
// Padding scale rows [M, round_up(M,128))
// are cleared word by word.
constexpr int kSmallQuantThreadsAll = 4096;       // threads of the cluster
constexpr int kSmallQuantElems = 16 * 8192;       // M*K up to this takes the one-cluster path

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int B, int CTAS>
__global__ void __launch_bounds__(kSmallQuantThreadsAll / CTAS) quantize_small_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx, int e4m3,
    const float* __restrict__ tscale_in, uint8_t* __restrict__ q, int64_t ldq, uint8_t* __restrict__ sf,
    float* __restrict__ tscale_out, int64_t sf_rows) {
  constexpr int kThreadsAll = kSmallQuantThreadsAll;
  constexpr int kThreads = kThreadsAll / CTAS;
  constexpr int kUPT = (kSmallQuantElems / B + kThreadsAll - 1) / kThreadsAll;   // blocks per thread
  __shared__ uint32_t red[kThreads / 32];
  __shared__ uint32_t cta_max[CTAS];
  const bool need_amax = e4m3 && !tscale_in;
  if (need_amax) cluster_arrive_relaxed();  // "started": no remote store before every CTA runs
  griddep_launch_dependents();              // the next kernel may set up meanwhile
  griddep_wait();                           // x may come from the previous kernel
  const uint32_t rank = cluster_ctarank();
  const int kb_per_row = static_cast<int>(K / B);
  const uint32_t g = rank * kThreads + threadIdx.x;
  const uint32_t units = static_cast<uint32_t>(M) * kb_per_row;
  // this thread's blocks, in registers
  uint32_t w[kUPT][B / 2];
  uint32_t m = 0;
#pragma unroll
  for (int t = 0; t < kUPT; ++t) {
    const uint32_t u = g + t * kThreadsAll;
    if (u < units) {
      const uint32_t r = u / kb_per_row, kb = u - r * kb_per_row;
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(r) * ldx + static_cast<int64_t>(kb) * B);
#pragma unroll
      for (int i = 0; i < B / 8; ++i) {
        const uint4 v = __ldg(src + i);
        w[t][4 * i] = v.x; w[t][4 * i + 1] = v.y; w[t][4 * i + 2] = v.z; w[t][4 * i + 3] = v.w;
      }
#pragma unroll
      for (int i = 0; i < B / 2; ++i) m = max(m, max(w[t][i] & 0x7FFFu, (w[t][i] >> 16) & 0x7FFFu));
    }
  }
  // padding scale rows: zero
  const int kb4 = kb_per_row / 4;
  const uint32_t pad_words = static_cast<uint32_t>(sf_rows - M) * kb4;
  for (uint32_t v = g; v < pad_words; v += kThreadsAll) {
    const int64_t pr = M + v / kb4;
    *reinterpret_cast<uint32_t*>(sf + sf_offset(pr, static_cast<int>(v % kb4) * 4, kb_per_row)) = 0u;
  }
  float s = 1.0f;
  if (e4m3 && tscale_in) s = *tscale_in;
  if (need_amax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    cluster_wait_acquire();                  // every CTA of the cluster is running
    __syncthreads();
    if (threadIdx.x < CTAS) {                // push this CTA's maximum into CTA threadIdx.x
      uint32_t mm = 0;
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) mm = max(mm, red[i]);
      st_cluster_u32(mapa_shared(smem_u32(&cta_max[rank]), threadIdx.x), mm);
    }
    __syncwarp();                            // the cluster barrier is warp-aligned
    cluster_sync_all();                      // all maxima everywhere; nothing remote after this
    uint32_t mm = 0;
#pragma unroll
    for (int i = 0; i < CTAS; ++i) mm = max(mm, cta_max[i]);
    const float amax = __uint_as_float(mm << 16);
    s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
  }
  if (tscale_out && rank == 0 && threadIdx.x == 0) *tscale_out = s;
#pragma unroll
  for (int t = 0; t < kUPT; ++t) {
    const uint32_t u = g + t * kThreadsAll;
    if (u < units) {
      const uint32_t r = u / kb_per_row, kb = u - r * kb_per_row;
      uint32_t qw[B / 8], sfb;
      quantize_block<B>(w[t], e4m3 != 0, s, qw, sfb);
      uint8_t* dst = q + static_cast<int64_t>(r) * ldq + static_cast<int64_t>(kb) * (B / 2);
      if (B == 32) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(qw[0], qw[1], qw[2], qw[3]);
      } else {
        *reinterpret_cast<uint2*>(dst) = make_uint2(qw[0], qw[1]);
      }
      sf[sf_offset(r, static_cast<int>(kb), kb_per_row)] = static_cast<uint8_t>(sfb);
    }
  }
}

// ------------------------------------------------------------------------------------
// Group prologue: validates offsets and writes tile_prefix[g] = sum over g' < g of
// ceil(rows_g' / 128), g = 0..E, and (when chunk_prefix is given) chunk_prefix[g] =
// sum over g' < g of ceil(tiles_g' / 2): the 256-row chunks the grouped kernel runs.
// Malformed offsets set MXC_ERR_DEVICE_INVALID and all-zero prefixes, so that the
// kernels that follow do no work.
// ------------------------------------------------------------------------------------
__global__ void group_prologue_kernel(const int32_t* __restrict__ offsets, int32_t E, int64_t M,
                                      int32_t* __restrict__ tile_prefix, int32_t* __restrict__ chunk_prefix) {
  __shared__ int bad;
  __shared__ int32_t tiles[kMaxGroups + 1];
  if (threadIdx.x == 0) bad = (offsets[0] != 0 || offsets[E] != M);
  __syncthreads();
  for (int g = threadIdx.x; g < E; g += blockDim.x) {
    const int32_t c = offsets[g + 1] - offsets[g];
    if (c < 0) bad = 1;
    tiles[g] = c > 0 ? (c + 127) / 128 : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t acc = 0, acc2 = 0;
    for (int g = 0; g < E; ++g) {
      tile_prefix[g] = bad ? 0 : acc;
      if (chunk_prefix) chunk_prefix[g] = bad ? 0 : acc2;
      acc += tiles[g];
      acc2 += (tiles[g] + 1) / 2;
    }
    tile_prefix[E] = bad ? 0 : acc;
    if (chunk_prefix) chunk_prefix[E] = bad ? 0 : acc2;
    if (bad) set_device_error(MXC_ERR_DEVICE_INVALID);
  }
}

// ------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------
cudaError_t launch_group_prologue(const int32_t* offsets, int32_t E, int64_t M, int32_t* tile_prefix,
                                  cudaStream_t stream, int32_t* chunk_prefix) {
  group_prologue_kernel<<<1, 256, 0, stream>>>(offsets, E, M, tile_prefix, chunk_prefix);
  return cudaGetLastError();
}

template <int B, int CTAS>
cudaError_t launch_quantize_small_ctas(const QuantizeArgs& a, const uint16_t* xp, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CTAS);
  cfg.blockDim = dim3(kSmallQuantThreadsAll / CTAS);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CTAS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int e4m3 = B == 16;
  const float* tin = e4m3 ? a.tscale_in : nullptr;
  cudaError_t err = cudaLaunchKernelEx(&cfg, quantize_small_kernel<B, CTAS>, xp, a.M, a.K, a.ldx, e4m3, tin, a.q,
                                       a.ldq, a.sf, a.tscale_out, a.sf_rows);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// A cluster of 16 CTAs (non-portable size) where the device schedules one, else 8.
template <int B>
cudaError_t launch_quantize_small(const QuantizeArgs& a, const uint16_t* xp, cudaStream_t stream) {
  static int use16 = -1;                     // decided once per process
  if (use16 < 0) {
    auto k = quantize_small_kernel<B, 16>;
    int n = 0;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(kSmallQuantThreadsAll / 16);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();                      // clear a refusal of the query
    use16 = n > 0 ? 1 : 0;
  }
  return use16 ? launch_quantize_small_ctas<B, 16>(a, xp, stream) : launch_quantize_small_ctas<B, 8>(a, xp, stream);
}

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream) {
  const bool e4m3 = a.fmt == MXC_FMT_E4M3_B16;
  const int B = e4m3 ? 16 : 32;
  unsigned int* amax_ws = reinterpret_cast<unsigned int*>(a.ws);
  if (!a.tile_prefix && a.M * a.K <= kSmallQuantElems) {
    const uint16_t* xp = reinterpret_cast<const uint16_t*>(a.x);
    if (e4m3) return launch_quantize_small<16>(a, xp, stream);
    return launch_quantize_small<32>(a, xp, stream);
  }
  if (e4m3 && !a.tscale_in) {
    cudaError_t err = cudaMemsetAsync(amax_ws, 0, sizeof(unsigned int), stream);
    if (err != cudaSuccess) return err;
    const int64_t chunks = a.M * (a.K / 8);
    const int threads = 256;
    const int64_t want = (chunks + threads - 1) / threads;
    const int blocks = static_cast<int>(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
    amax_kernel<<<blocks, threads, 0, stream>>>(reinterpret_cast<const uint16_t*>(a.x), a.M, a.K, a.ldx,
                                                amax_ws);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  const int64_t units = a.sf_rows * (a.K / B);
  const int threads = 256;
  const int64_t want = (units + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  if (e4m3) {
    quantize_kernel<16><<<blocks, threads, 0, stream>>>(
        reinterpret_cast<const uint16_t*>(a.x), a.M, a.K, a.ldx, 1, a.tscale_in, amax_ws, a.q, a.ldq,
        a.sf, a.tscale_out, a.sf_rows, a.offsets, a.tile_prefix, a.n_groups);
  } else {
    quantize_kernel<32><<<blocks, threads, 0, stream>>>(
        reinterpret_cast<const uint16_t*>(a.x), a.M, a.K, a.ldx, 0, nullptr, nullptr, a.q, a.ldq, a.sf,
        a.tscale_out, a.sf_rows, a.offsets, a.tile_prefix, a.n_groups);
  }
  return cudaGetLastError();
}

}  // namespace mxc
