// mxc_internal.h -- declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "mxc.h"

namespace mxc {

constexpr int kMaxGroups = 256;     // experts per grouped call (kernel-parameter table size)
constexpr int kTileN = 128;         // output channels per CTA tile (MMA M)
constexpr int kStageK = 256;        // input channels per pipeline stage (one 128-byte FP4 row)

struct QuantizeArgs {
  const void* x;
  int64_t M, K, ldx;
  mxc_format fmt;
  const float* tscale_in;
  uint8_t* q;
  int64_t ldq;
  uint8_t* sf;
  float* tscale_out;
  void* ws;
  int64_t sf_rows;              // scale rows to write (dense: round_up(M,128); grouped: bound)
  const int32_t* offsets;       // grouped mode only
  const int32_t* tile_prefix;   // grouped mode only (device, from the group prologue)
  int32_t n_groups;
};

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream);
cudaError_t launch_group_prologue(const int32_t* offsets, int32_t E, int64_t M, int32_t* tile_prefix,
                                  cudaStream_t stream, int32_t* chunk_prefix = nullptr);

// Linear-layer launch descriptions (filled by the host API after validation).
struct LinearArgs {
  // activation
  const uint8_t* a_q;
  const uint8_t* a_sf;
  const float* a_tscale;
  int64_t M, K, ldq;
  // weight: VQ (idx/cb/scales|sidx+scb) or native (w_q + w_sf)
  int wsrc;                     // 0 VQ direct scales, 1 VQ scale-VQ, 2 native FP4
  int fmt;                      // 0 E8M0-B32, 1 E4M3-B16
  int64_t N, qn, qk;
  const uint8_t* w_idx;
  const uint16_t* w_cb;
  const uint8_t* w_sf;
  const uint8_t* w_sidx;
  const uint8_t* w_scb;
  const uint8_t* w_q;           // native
  int64_t w_ldq;                // native
  float w_tscale;
  int w_ds;                     // PreScale+ scale group
  const float* w_tscale_dev;    // native (device) or null
  // output
  void* y;
  int64_t ldy;
  int out_bf16;
  // workspace: [split-K arrival counters, kSplitkCtrBytes][the decoded weight, decode once]
  // [split-K partial tiles]; ws_used = bytes past the counter area already taken
  void* ws;
  size_t ws_bytes;
  size_t ws_used;
};

struct MoeArgs {
  LinearArgs base;              // shapes, format, activation, output; weight pointers unused
  const int32_t* offsets;
  int32_t E;
  const mxc_weight* experts;    // host array
  // gate/up with SwiGLU: h = SiLU(gate) * up quantized into the down projection's
  // activation instead of writing y
  int swiglu;
  uint8_t* h_q;
  int64_t ldh;
  uint8_t* h_sf;
  const float* h_tscale;
};

struct DecodeArgs {
  int wsrc, fmt;
  int64_t N, K, qn, qk;
  const uint8_t* w_idx;
  const uint16_t* w_cb;
  const uint8_t* w_sf;
  const uint8_t* w_sidx;
  const uint8_t* w_scb;
  int ds;                       // PreScale+ scale group
  uint8_t* q_out;
  int64_t ldq;
  uint8_t* sf_out;
};

mxc_status run_linear(const LinearArgs& a, cudaStream_t stream);
mxc_status run_moe_linear(const MoeArgs& a, cudaStream_t stream);
mxc_status run_decode_weight(const DecodeArgs& a, cudaStream_t stream);

size_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt);
size_t linear_workspace_bytes_for(int64_t M, int64_t N, int64_t K, int fmt, int64_t qn, int64_t qk);
size_t moe_workspace_bytes(int64_t M, int32_t E, int64_t N, int64_t K, int fmt);

}  // namespace mxc
