// mxc_lib.cu -- the C ABI of the MXCode W4A4 library (declared in include/mxc.h).
//
// The whole library is one translation unit (this file includes the kernels), so
// the per-device error word is an ordinary module global.  Entry points validate
// their arguments on the host, then enqueue kernels on the caller's stream.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "act_quant.cuh"
#include "linear.cuh"
#include "mxc.h"

using namespace mxc;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int block_of(mxc_format f) { return f == MXC_FMT_E8M0_B32 ? 32 : 16; }

mxc_status check_format(mxc_format f) {
  if (f == MXC_FMT_E8M0_B32 || f == MXC_FMT_E4M3_B16) return MXC_OK;
  if (f == MXC_FMT_UE5M3_B16) return MXC_ERR_UNSUPPORTED;
  return MXC_ERR_INVALID_ARG;
}

mxc_status check_device() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXC_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MXC_ERR_NO_DEVICE;
  return major == 10 ? MXC_OK : MXC_ERR_NO_DEVICE;
}

// Resolved QBlock sizes; checks the divisibility the kernels rely on.
mxc_status resolve_qblock(int64_t N, int64_t K, int64_t qn_in, int64_t qk_in, int64_t* qn, int64_t* qk) {
  *qn = qn_in ? qn_in : N;
  *qk = qk_in ? qk_in : K;
  if (*qn <= 0 || *qk <= 0) return MXC_ERR_INVALID_ARG;
  // 64 rows or 64 input channels (down to 64 x 64), 128 input channels, or multiples
  // of the 128-row tile and the 256-channel stage
  if ((*qn != 64 && *qn % kTileN) || N % *qn) return MXC_ERR_ALIGNMENT;
  if (!(*qk == 64 || *qk == 128 || *qk % kStageK == 0) || K % *qk) return MXC_ERR_ALIGNMENT;
  return MXC_OK;
}

// Where a VQ weight's block scales come from, for the kernels.
int wsrc_of(mxc_strategy st) {
  return st == MXC_PRESCALE_PLUS ? WSRC_VQ_SVQ : st == MXC_POSTSCALE_QB ? WSRC_VQ_QBS : WSRC_VQ_DIRECT;
}

mxc_status check_shape(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0) return MXC_ERR_INVALID_ARG;
  if (N % kTileN || K % kStageK) return MXC_ERR_ALIGNMENT;
  if (N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return MXC_ERR_UNSUPPORTED;
  return MXC_OK;
}

// PreScale+ scale group: 0 means 8 (Table 4 caption); 16 and 32 are the higher
// scale-compression ratios of Figure 3; K must hold whole groups.
mxc_status resolve_scale_group(mxc_strategy strategy, mxc_format fmt, int64_t K, int32_t sg, int* ds) {
  *ds = 8;
  if (strategy != MXC_PRESCALE_PLUS) return MXC_OK;
  *ds = sg ? sg : 8;
  if (*ds != 8 && *ds != 16 && *ds != 32) return MXC_ERR_INVALID_ARG;
  if (K % (static_cast<int64_t>(*ds) * block_of(fmt))) return MXC_ERR_ALIGNMENT;
  return MXC_OK;
}

mxc_status check_weight_common(mxc_strategy strategy, mxc_format fmt, int64_t N, int64_t K, int64_t qn, int64_t qk,
                               int32_t sg, int64_t* rqn, int64_t* rqk, int* ds) {
  mxc_status s = check_format(fmt);
  if (s != MXC_OK) return s;
  if (strategy != MXC_POSTSCALE && strategy != MXC_PRESCALE && strategy != MXC_PRESCALE_PLUS &&
      strategy != MXC_POSTSCALE_QB)
    return MXC_ERR_INVALID_ARG;
  if ((s = check_shape(N, K)) != MXC_OK) return s;
  if ((s = resolve_scale_group(strategy, fmt, K, sg, ds)) != MXC_OK) return s;
  return resolve_qblock(N, K, qn, qk, rqn, rqk);
}

mxc_status check_device_weight(const mxc_weight* w, int64_t* qn, int64_t* qk, int* ds) {
  if (!w) return MXC_ERR_INVALID_ARG;
  mxc_status s = check_weight_common(w->strategy, w->fmt, w->N, w->K, w->qn, w->qk, w->scale_group, qn, qk, ds);
  if (s != MXC_OK) return s;
  if (!w->idx || !w->cb) return MXC_ERR_INVALID_ARG;
  if (!aligned16(w->idx) || !aligned16(w->cb)) return MXC_ERR_ALIGNMENT;
  if (w->strategy == MXC_PRESCALE_PLUS) {
    if (!w->sidx || !w->scb) return MXC_ERR_INVALID_ARG;
    if (!aligned16(w->sidx) || !aligned16(w->scb)) return MXC_ERR_ALIGNMENT;
  } else {
    if (!w->scales) return MXC_ERR_INVALID_ARG;
    if (!aligned16(w->scales)) return MXC_ERR_ALIGNMENT;
  }
  return MXC_OK;
}

mxc_status check_mx_tensor(const mxc_mx_tensor* t) {
  if (!t || !t->q || !t->sf) return MXC_ERR_INVALID_ARG;
  mxc_status s = check_format(t->fmt);
  if (s != MXC_OK) return s;
  if (t->rows < 0 || t->K <= 0) return MXC_ERR_INVALID_ARG;
  if (t->K % kStageK) return MXC_ERR_ALIGNMENT;
  if (t->ldq < t->K / 2 || t->ldq % 16) return MXC_ERR_ALIGNMENT;
  if (!aligned16(t->q) || !aligned16(t->sf)) return MXC_ERR_ALIGNMENT;
  if (t->rows > (int64_t(1) << 30)) return MXC_ERR_UNSUPPORTED;
  return MXC_OK;
}

mxc_status check_output(const void* y, int64_t ldy, int64_t N, mxc_dtype dt) {
  if (!y) return MXC_ERR_INVALID_ARG;
  if (dt != MXC_OUT_F32 && dt != MXC_OUT_BF16) return MXC_ERR_INVALID_ARG;
  if (ldy < N) return MXC_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(y) & (dt == MXC_OUT_F32 ? 3u : 1u)) return MXC_ERR_ALIGNMENT;
  return MXC_OK;
}

inline size_t sf_bytes(int64_t rows, int64_t K, mxc_format fmt) {
  return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(K / block_of(fmt));
}

inline size_t sf_off_host(int64_t r, int64_t kb, int64_t kb_per_row) {
  return static_cast<size_t>((r / 128) * (kb_per_row / 4) + kb / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 +
         (kb % 4);
}

// Runs the pipelines' bounded mbarrier wait on a barrier that nothing arrives
// at: the wait gives up after `limit` clocks, records MXC_ERR_TIMEOUT and the
// kernel returns (nothing is in flight).
__global__ void wait_timeout_probe_kernel(long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait_limit(&bar, 0, limit);
  }
}

}  // namespace

extern "C" {

const char* mxc_status_string(mxc_status s) {
  switch (s) {
    case MXC_OK: return "ok";
    case MXC_ERR_INVALID_ARG: return "invalid argument";
    case MXC_ERR_UNSUPPORTED: return "unsupported";
    case MXC_ERR_ALIGNMENT: return "shape or alignment requirement not met";
    case MXC_ERR_WORKSPACE: return "workspace missing or too small";
    case MXC_ERR_CUDA: return "CUDA call failed";
    case MXC_ERR_DEVICE_INVALID: return "device found malformed data";
    case MXC_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MXC_ERR_NO_DEVICE: return "no sm_100 device is current";
  }
  return "unknown status";
}

int mxc_version(void) { return 100; }

size_t mxc_sf_bytes(int64_t rows, int64_t K, mxc_format fmt) {
  if (check_format(fmt) != MXC_OK || rows < 0 || K <= 0) return 0;
  return sf_bytes(rows, K, fmt);
}

mxc_status mxc_packed_weight_sizes(const mxc_weight_host* w, mxc_packed_sizes* out) {
  if (!w || !out) return MXC_ERR_INVALID_ARG;
  int64_t qn, qk;
  int ds;
  mxc_status s = check_weight_common(w->strategy, w->fmt, w->N, w->K, w->qn, w->qk, w->scale_group, &qn, &qk, &ds);
  if (s != MXC_OK) return s;
  const int B = block_of(w->fmt);
  out->idx = static_cast<size_t>(w->N) * (w->K / 4);
  out->cb = static_cast<size_t>(w->N / qn) * (w->K / qk) * 256 * sizeof(uint16_t);
  if (w->strategy == MXC_PRESCALE_PLUS) {
    out->scales = 0;
    out->sidx = static_cast<size_t>(w->N) * (w->K / (static_cast<int64_t>(ds) * B));
    out->scb = 256 * static_cast<size_t>(ds);
  } else if (w->strategy == MXC_POSTSCALE_QB) {
    out->scales = static_cast<size_t>(w->N / qn) * static_cast<size_t>(w->K / qk);
    out->sidx = 0;
    out->scb = 0;
  } else {
    out->scales = sf_bytes(w->N, w->K, w->fmt);
    out->sidx = 0;
    out->scb = 0;
  }
  return MXC_OK;
}

mxc_status mxc_pack_weight(const mxc_weight_host* w, uint8_t* idx_out, uint8_t* scales_out, uint8_t* sidx_out) {
  mxc_packed_sizes sz;
  mxc_status s = mxc_packed_weight_sizes(w, &sz);
  if (s != MXC_OK) return s;
  const int64_t N = w->N, K = w->K, KS = K / kStageK;
  const int B = block_of(w->fmt);
  if (idx_out) {
    if (!w->idx) return MXC_ERR_INVALID_ARG;
    for (int64_t nt = 0; nt < N / kTileN; ++nt)
      for (int64_t ks = 0; ks < KS; ++ks)
        for (int64_t c = 0; c < 4; ++c)         // K-quarter slabs of 16 index bytes per row
          for (int64_t r = 0; r < kTileN; ++r)
            std::memcpy(idx_out + ((nt * KS + ks) * 4 + c) * 2048 + r * 16,
                        w->idx + (nt * kTileN + r) * (K / 4) + ks * 64 + c * 16, 16);
  }
  if (w->strategy == MXC_PRESCALE_PLUS) {
    if (sidx_out) {
      if (!w->sidx) return MXC_ERR_INVALID_ARG;
      // units of the band's indices: a 256-channel stage holding G = 256/(ds*B)
      // groups of each row when ds*B <= 256, else one group (G = 1)
      const int ds = w->scale_group ? w->scale_group : 8;
      const int64_t row = K / (static_cast<int64_t>(ds) * B);
      const int64_t G = ds * B <= kStageK ? kStageK / (ds * B) : 1, U = row / G;
      for (int64_t nt = 0; nt < N / kTileN; ++nt)
        for (int64_t u = 0; u < U; ++u)
          for (int64_t r = 0; r < kTileN; ++r)
            std::memcpy(sidx_out + ((nt * U + u) * kTileN + r) * G, w->sidx + (nt * kTileN + r) * row + u * G, G);
    }
  } else if (scales_out && w->strategy == MXC_POSTSCALE_QB) {
    if (!w->scales) return MXC_ERR_INVALID_ARG;
    std::memcpy(scales_out, w->scales, sz.scales);   // [N/qn][K/qk]: already the packed layout
  } else if (scales_out) {
    if (!w->scales) return MXC_ERR_INVALID_ARG;
    const int64_t KB = K / B;
    std::memset(scales_out, 0, sz.scales);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t kb = 0; kb < KB; ++kb) scales_out[sf_off_host(n, kb, KB)] = w->scales[n * KB + kb];
  }
  return MXC_OK;
}

size_t mxc_quantize_act_workspace_bytes(int64_t /*M*/, int64_t /*K*/, mxc_format /*fmt*/) { return 256; }

size_t mxc_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, mxc_format fmt) {
  if (check_format(fmt) != MXC_OK || check_shape(N, K) != MXC_OK || M < 0) return 0;
  return linear_workspace_bytes(M, N, K, fmt);
}

size_t mxc_linear_workspace_bytes_for(const mxc_weight* w, int64_t M) {
  int64_t qn, qk;
  int ds;
  if (!w || M < 0 || check_weight_common(w->strategy, w->fmt, w->N, w->K, w->qn, w->qk, w->scale_group, &qn, &qk,
                                         &ds) != MXC_OK)
    return 0;
  return linear_workspace_bytes_for(M, w->N, w->K, w->fmt == MXC_FMT_E8M0_B32 ? FMT_E8M0 : FMT_E4M3, qn, qk);
}

size_t mxc_moe_workspace_bytes(int64_t M, int32_t E, int64_t N, int64_t K, mxc_format fmt) {
  if (E <= 0) return 0;
  return moe_workspace_bytes(M, E, N, K, fmt);
}

int64_t mxc_grouped_sf_rows_bound(int64_t M, int32_t E) {
  return (M + 127) / 128 * 128 + static_cast<int64_t>(E > 0 ? E : 0) * 128;
}

static mxc_status quantize_common(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxc_format fmt,
                                  const int32_t* d_offsets, int32_t E, const float* act_tscale_in, uint8_t* q_out,
                                  int64_t ldq, uint8_t* sf_out, float* act_tscale_out, void* ws, size_t ws_bytes,
                                  mxc_stream_t stream) {
  mxc_status s = check_format(fmt);
  if (s != MXC_OK) return s;
  if (M < 0 || K <= 0 || ldx < K || ldq < K / 2) return MXC_ERR_INVALID_ARG;
  if (K % kStageK || ldq % 16 || ldx % 8) return MXC_ERR_ALIGNMENT;
  if (M > (int64_t(1) << 30)) return MXC_ERR_UNSUPPORTED;
  if (M == 0) return MXC_OK;
  if (!x_bf16 || !q_out || !sf_out) return MXC_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(q_out) || !aligned16(sf_out)) return MXC_ERR_ALIGNMENT;
  const bool e4m3 = fmt == MXC_FMT_E4M3_B16;
  if (e4m3 && !act_tscale_out) return MXC_ERR_INVALID_ARG;
  const size_t need = mxc_quantize_act_workspace_bytes(M, K, fmt) + (d_offsets ? (static_cast<size_t>(E) + 1) * 4 : 0);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MXC_ERR_WORKSPACE;
  if ((s = check_device()) != MXC_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  QuantizeArgs a{};
  a.x = x_bf16;
  a.M = M;
  a.K = K;
  a.ldx = ldx;
  a.fmt = fmt;
  a.tscale_in = e4m3 ? act_tscale_in : nullptr;
  a.q = q_out;
  a.ldq = ldq;
  a.sf = sf_out;
  a.tscale_out = act_tscale_out;
  a.ws = ws;
  if (d_offsets) {
    if (E <= 0 || E > kMaxGroups) return MXC_ERR_INVALID_ARG;
    int32_t* tile_prefix = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + 256);
    if (launch_group_prologue(d_offsets, E, M, tile_prefix, st) != cudaSuccess) return MXC_ERR_CUDA;
    a.offsets = d_offsets;
    a.tile_prefix = tile_prefix;
    a.n_groups = E;
    a.sf_rows = mxc_grouped_sf_rows_bound(M, E);
  } else {
    a.sf_rows = (M + 127) / 128 * 128;
  }
  return launch_quantize(a, st) == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
}

mxc_status mxc_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxc_format fmt,
                            const float* act_tscale_in, uint8_t* q_out, int64_t ldq, uint8_t* sf_out,
                            float* act_tscale_out, void* ws, size_t ws_bytes, mxc_stream_t stream) {
  return quantize_common(x_bf16, M, K, ldx, fmt, nullptr, 0, act_tscale_in, q_out, ldq, sf_out, act_tscale_out, ws,
                         ws_bytes, stream);
}

mxc_status mxc_quantize_act_grouped(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxc_format fmt,
                                    const int32_t* d_offsets, int32_t E, const float* act_tscale_in, uint8_t* q_out,
                                    int64_t ldq, uint8_t* sf_out, float* act_tscale_out, void* ws, size_t ws_bytes,
                                    mxc_stream_t stream) {
  if (!d_offsets) return MXC_ERR_INVALID_ARG;
  return quantize_common(x_bf16, M, K, ldx, fmt, d_offsets, E, act_tscale_in, q_out, ldq, sf_out, act_tscale_out, ws,
                         ws_bytes, stream);
}

static void fill_activation(LinearArgs& L, const mxc_mx_tensor* a) {
  L.a_q = a->q;
  L.a_sf = a->sf;
  L.a_tscale = a->tscale;
  L.M = a->rows;
  L.K = a->K;
  L.ldq = a->ldq;
  L.fmt = a->fmt == MXC_FMT_E8M0_B32 ? FMT_E8M0 : FMT_E4M3;
}

mxc_status mxc_linear(const mxc_mx_tensor* a, const mxc_weight* w, void* y, int64_t ldy, mxc_dtype y_dtype, void* ws,
                      size_t ws_bytes, mxc_stream_t stream) {
  mxc_status s = check_mx_tensor(a);
  if (s != MXC_OK) return s;
  int64_t qn, qk;
  int ds;
  if ((s = check_device_weight(w, &qn, &qk, &ds)) != MXC_OK) return s;
  if (a->fmt != w->fmt || a->K != w->K) return MXC_ERR_INVALID_ARG;
  if ((s = check_output(y, ldy, w->N, y_dtype)) != MXC_OK) return s;
  if (a->rows == 0) return MXC_OK;
  if ((s = check_device()) != MXC_OK) return s;
  LinearArgs L{};
  fill_activation(L, a);
  L.wsrc = wsrc_of(w->strategy);
  L.N = w->N;
  L.qn = qn;
  L.qk = qk;
  L.w_idx = w->idx;
  L.w_cb = w->cb;
  L.w_sf = w->scales;
  L.w_sidx = w->sidx;
  L.w_scb = w->scb;
  L.w_tscale = w->w_tscale;
  L.w_ds = ds;
  L.y = y;
  L.ldy = ldy;
  L.out_bf16 = y_dtype == MXC_OUT_BF16;
  L.ws = ws;
  L.ws_bytes = ws_bytes;
  return run_linear(L, reinterpret_cast<cudaStream_t>(stream));
}

mxc_status mxc_native_linear(const mxc_mx_tensor* a, const mxc_mx_tensor* w, void* y, int64_t ldy, mxc_dtype y_dtype,
                             void* ws, size_t ws_bytes, mxc_stream_t stream) {
  mxc_status s = check_mx_tensor(a);
  if (s != MXC_OK) return s;
  if ((s = check_mx_tensor(w)) != MXC_OK) return s;
  if (a->fmt != w->fmt || a->K != w->K) return MXC_ERR_INVALID_ARG;
  if ((s = check_shape(w->rows, w->K)) != MXC_OK) return s;
  if ((s = check_output(y, ldy, w->rows, y_dtype)) != MXC_OK) return s;
  if (a->rows == 0) return MXC_OK;
  if ((s = check_device()) != MXC_OK) return s;
  LinearArgs L{};
  fill_activation(L, a);
  L.wsrc = WSRC_NATIVE;
  L.N = w->rows;
  L.qn = w->rows;
  L.qk = w->K;
  L.w_q = w->q;
  L.w_ldq = w->ldq;
  L.w_sf = w->sf;
  L.w_tscale = 1.0f;
  L.w_tscale_dev = w->tscale;
  L.y = y;
  L.ldy = ldy;
  L.out_bf16 = y_dtype == MXC_OUT_BF16;
  L.ws = ws;
  L.ws_bytes = ws_bytes;
  return run_linear(L, reinterpret_cast<cudaStream_t>(stream));
}

// Argument checks shared by the grouped entry points, in one order of precedence
// (activation, offsets and expert table, each expert, consistency); the output is
// checked by the caller.
static mxc_status moe_prepare_inputs(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                                     int32_t E, MoeArgs* m) {
  mxc_status s = check_mx_tensor(a);
  if (s != MXC_OK) return s;
  if (!d_offsets || !experts || E <= 0) return MXC_ERR_INVALID_ARG;
  if (E > kMaxGroups) return MXC_ERR_UNSUPPORTED;
  int64_t qn, qk;
  int ds;
  if ((s = check_device_weight(&experts[0], &qn, &qk, &ds)) != MXC_OK) return s;
  for (int32_t e = 1; e < E; ++e) {
    const mxc_weight& w = experts[e];
    int64_t qn2, qk2;
    int ds2;
    if ((s = check_device_weight(&w, &qn2, &qk2, &ds2)) != MXC_OK) return s;
    if (w.strategy != experts[0].strategy || w.fmt != experts[0].fmt || w.N != experts[0].N ||
        w.K != experts[0].K || qn2 != qn || qk2 != qk || ds2 != ds)
      return MXC_ERR_INVALID_ARG;
  }
  const mxc_weight& w0 = experts[0];
  if (a->fmt != w0.fmt || a->K != w0.K) return MXC_ERR_INVALID_ARG;
  if (small_qblock(qn, qk)) return MXC_ERR_UNSUPPORTED;   // grouped kernels decode in the GEMM
  *m = MoeArgs{};
  fill_activation(m->base, a);
  m->base.wsrc = wsrc_of(w0.strategy);
  m->base.N = w0.N;
  m->base.qn = qn;
  m->base.qk = qk;
  m->offsets = d_offsets;
  m->E = E;
  m->experts = experts;
  return MXC_OK;
}

static mxc_status moe_prepare(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts, int32_t E,
                              void* y, int64_t ldy, mxc_dtype y_dtype, MoeArgs* m) {
  mxc_status s = moe_prepare_inputs(a, d_offsets, experts, E, m);
  if (s != MXC_OK) return s;
  if ((s = check_output(y, ldy, m->base.N, y_dtype)) != MXC_OK) return s;
  m->base.y = y;
  m->base.ldy = ldy;
  m->base.out_bf16 = y_dtype == MXC_OUT_BF16;
  return MXC_OK;
}

mxc_status mxc_moe_linear(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts, int32_t E,
                          void* y, int64_t ldy, mxc_dtype y_dtype, void* ws, size_t ws_bytes, mxc_stream_t stream) {
  MoeArgs m;
  mxc_status s = moe_prepare(a, d_offsets, experts, E, y, ldy, y_dtype, &m);
  if (s != MXC_OK) return s;
  if (a->rows == 0) return MXC_OK;
  if ((s = check_device()) != MXC_OK) return s;
  m.base.ws = ws;
  m.base.ws_bytes = ws_bytes;
  return run_moe_linear(m, reinterpret_cast<cudaStream_t>(stream));
}

mxc_status mxc_moe_gate_up_swiglu(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                                  int32_t E, const float* h_tscale_in, uint8_t* h_q, int64_t ldh, uint8_t* h_sf,
                                  void* ws, size_t ws_bytes, mxc_stream_t stream) {
  MoeArgs m;
  mxc_status s = moe_prepare_inputs(a, d_offsets, experts, E, &m);
  if (s != MXC_OK) return s;
  const int64_t F = m.base.N / 2;
  if (m.base.N % 2 || F % kTileN) return MXC_ERR_ALIGNMENT;
  if (!h_q || !h_sf) return MXC_ERR_INVALID_ARG;
  if (ldh < F / 2 || ldh % 16 || !aligned16(h_q) || !aligned16(h_sf)) return MXC_ERR_ALIGNMENT;
  if (a->fmt == MXC_FMT_E4M3_B16 && !h_tscale_in) return MXC_ERR_INVALID_ARG;
  if (a->rows == 0) return MXC_OK;
  if ((s = check_device()) != MXC_OK) return s;
  m.base.ws = ws;
  m.base.ws_bytes = ws_bytes;
  m.swiglu = 1;
  m.h_q = h_q;
  m.ldh = ldh;
  m.h_sf = h_sf;
  m.h_tscale = h_tscale_in;
  return run_moe_linear(m, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Allocation-free MoE entry point: the expert tile and chunk tables (E+1 int32 each)
// live in a fixed module-global array instead of a caller workspace.
// ------------------------------------------------------------------------------------
namespace {

// The largest tables the grouped kernels use (256 experts), in whole 256-byte units,
// exactly the workspace size mxc_moe_workspace_bytes reports for 256 experts.
constexpr size_t kNoallocScratchBytes = (2 * static_cast<size_t>(kMaxGroups + 1) * sizeof(int32_t) + 255) / 256 * 256;
static __device__ __align__(256) int32_t g_moe_noalloc_scratch[kNoallocScratchBytes / sizeof(int32_t)];

constexpr int kMaxDevices = 64;
std::atomic<int32_t*> g_noalloc_ptr[kMaxDevices];

// Device address of g_moe_noalloc_scratch on the current device (looked up once
// per device; a host-side name of a __device__ array is not a device address).
mxc_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MXC_ERR_NO_DEVICE;
  int32_t* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_moe_noalloc_scratch) != cudaSuccess || !addr) return MXC_ERR_CUDA;
    p = static_cast<int32_t*>(addr);
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MXC_OK;
}

}  // namespace

extern "C" {

mxc_status mxc_moe_linear_noalloc(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                                  int32_t E, void* y, int64_t ldy, mxc_dtype y_dtype, mxc_stream_t stream) {
  MoeArgs m;
  mxc_status s = moe_prepare(a, d_offsets, experts, E, y, ldy, y_dtype, &m);
  if (s != MXC_OK) return s;
  if (a->rows == 0) return MXC_OK;
  if ((s = check_device()) != MXC_OK) return s;
  const size_t need = mxc_moe_workspace_bytes(a->rows, E, m.base.N, m.base.K, a->fmt);
  if (need > kNoallocScratchBytes) return MXC_ERR_UNSUPPORTED;   // cannot happen for E <= 256
  int32_t* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != MXC_OK) return s;
  m.base.ws = scratch;
  m.base.ws_bytes = kNoallocScratchBytes;
  return run_moe_linear(m, reinterpret_cast<cudaStream_t>(stream));
}

mxc_status mxc_decode_weight(const mxc_weight* w, uint8_t* q_out, int64_t ldq, uint8_t* sf_out, mxc_stream_t stream) {
  int64_t qn, qk;
  int ds;
  mxc_status s = check_device_weight(w, &qn, &qk, &ds);
  if (s != MXC_OK) return s;
  if (!q_out || !sf_out) return MXC_ERR_INVALID_ARG;
  if (ldq < w->K / 2 || ldq % 16 || !aligned16(q_out) || !aligned16(sf_out)) return MXC_ERR_ALIGNMENT;
  if ((s = check_device()) != MXC_OK) return s;
  DecodeArgs d{};
  d.wsrc = wsrc_of(w->strategy);
  d.fmt = w->fmt == MXC_FMT_E8M0_B32 ? FMT_E8M0 : FMT_E4M3;
  d.N = w->N;
  d.K = w->K;
  d.qn = qn;
  d.qk = qk;
  d.w_idx = w->idx;
  d.w_cb = w->cb;
  d.w_sf = w->scales;
  d.w_sidx = w->sidx;
  d.w_scb = w->scb;
  d.ds = ds;
  d.q_out = q_out;
  d.ldq = ldq;
  d.sf_out = sf_out;
  return run_decode_weight(d, reinterpret_cast<cudaStream_t>(stream));
}

mxc_status mxc_selftest_wait_timeout(int64_t limit_cycles, mxc_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > kWaitLimitCycles) return MXC_ERR_INVALID_ARG;
  mxc_status s = check_device();
  if (s != MXC_OK) return s;
  wait_timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return cudaGetLastError() == cudaSuccess ? MXC_OK : MXC_ERR_CUDA;
}

mxc_status mxc_get_device_error(mxc_stream_t stream) {
  mxc_status s = check_device();
  if (s != MXC_OK) return s;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MXC_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_mxc_device_error, sizeof(v)) != cudaSuccess) return MXC_ERR_CUDA;
  if (v) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_mxc_device_error, &z, sizeof(z)) != cudaSuccess) return MXC_ERR_CUDA;
  }
  return static_cast<mxc_status>(v);
}

}  // extern "C"
