// qvae.cu -- host side of libqvae: argument checks, tiling choice, tensor-map
// encoding, launches, and the extern "C" entry points declared in qvae.h.
// All kernels live in one translation unit so they share the device error word.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/qvae.h"
#include "conv.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

using qvae::ConvArgs;

thread_local std::string t_last_error;
uint64_t g_wait_limit_ns = 2000000000ull;
int32_t g_force[5] = {0, 0, 0, 0, 0};  // BW, MS, NT, SA, SB

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
bool g_conv_attr_set[kMaxDevices][2] = {};

constexpr int kSmemLimit = 232448;  // dynamic shared memory per block on sm_100

int cuda_fail(cudaError_t e, const char* what) {
  char buf[256];
  std::snprintf(buf, sizeof buf, "%s: %s", what, cudaGetErrorString(e));
  t_last_error = buf;
  return QVAE_ERR_CUDA;
}

#define QVAE_CUDA(call)                                  \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);  \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device(int* dev) {
  QVAE_CUDA(cudaGetDevice(dev));
  if (*dev < 0 || *dev >= kMaxDevices) return QVAE_ERR_UNSUPPORTED;
  return QVAE_OK;
}

int sm_count(int dev, int* out) {
  if (g_sm_count[dev] == 0) {
    int n = 0;
    QVAE_CUDA(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
    g_sm_count[dev] = n;
  }
  *out = g_sm_count[dev];
  return QVAE_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// ------------------------------------------------------------------ tiling

struct Tiling {
  int BW, BH, MS, NT, SA, SB, acc_stages;
  uint32_t a_stage_bytes, b_stage_bytes, tmem_cols, smem_bytes;
  int tiles_w, tiles_h, tiles_n, num_tiles;
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

uint32_t smem_needed(const Tiling& t) {
  const uint32_t bars = 8 * qvae::kMaxStages * 4 + 16 + 16 + 8;
  return 1024 + t.SA * t.a_stage_bytes + t.SB * t.b_stage_bytes + bars + 16 + 4 * 2 * t.NT * 4;
}

int choose_nt(int Cout, int forced) {
  if (forced) return (forced % 32 == 0 && forced <= 256 && Cout % forced == 0) ? forced : 0;
  for (int n = static_cast<int>(ceil_div(Cout, 256)); n <= Cout / 32; ++n)
    if (Cout % n == 0 && (Cout / n) % 32 == 0) return Cout / n;
  return 0;
}

int make_tiling(const qvae_shape& s, Tiling* t) {
  t->NT = choose_nt(s.Cout, g_force[2]);
  if (t->NT == 0) return QVAE_ERR_SHAPE;
  t->MS = g_force[1] ? g_force[1] : 2;
  if (t->MS != 1 && t->MS != 2) return QVAE_ERR_ARG;
  // Tile width: least padded area, then the narrower tile (less halo per box).
  static const int kWidths[5] = {16, 32, 8, 64, 128};
  int best_bw = 0;
  int64_t best_area = 0;
  for (int bw : kWidths) {
    if (g_force[0] && bw != g_force[0]) continue;
    const int rows = t->MS * (128 / bw);
    const int64_t area = ceil_div(s.W, bw) * bw * ceil_div(s.H, rows) * rows;
    if (best_bw == 0 || area < best_area) { best_bw = bw; best_area = area; }
  }
  if (best_bw == 0) return QVAE_ERR_ARG;
  t->BW = best_bw;
  t->BH = 128 / best_bw;
  t->a_stage_bytes = static_cast<uint32_t>(t->MS * t->BH + 2) * t->BW * 128u;
  t->b_stage_bytes = static_cast<uint32_t>(t->NT) * 128u;
  const int acc_cols = t->MS * t->NT;
  t->acc_stages = (2 * acc_cols <= 512) ? 2 : 1;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(t->acc_stages * acc_cols)) cols <<= 1;
  t->tmem_cols = cols;
  if (g_force[3] || g_force[4]) {
    t->SA = g_force[3] ? g_force[3] : 2;
    t->SB = g_force[4] ? g_force[4] : 4;
    if (t->SA < 1 || t->SA > qvae::kMaxStages || t->SB < 1 || t->SB > qvae::kMaxStages) return QVAE_ERR_ARG;
  } else {
    // Deepest pipeline that fits, about three weight stages per activation stage.
    Tiling best = *t;
    best.SA = 0;
    for (int sa = 4; sa >= 2 && best.SA == 0; --sa) {
      Tiling u = *t;
      u.SA = sa;
      for (u.SB = 8; u.SB >= 3 && smem_needed(u) > kSmemLimit; --u.SB) {}
      if (smem_needed(u) <= kSmemLimit && u.SB >= std::min(8, 3 * sa - 1)) best = u;
    }
    if (best.SA == 0) {
      best = *t;
      best.SA = 2;
      for (best.SB = 8; best.SB > 2 && smem_needed(best) > kSmemLimit; --best.SB) {}
    }
    *t = best;
  }
  t->smem_bytes = smem_needed(*t);
  if (t->smem_bytes > kSmemLimit) return QVAE_ERR_UNSUPPORTED;
  t->tiles_w = static_cast<int>(ceil_div(s.W, t->BW));
  t->tiles_h = static_cast<int>(ceil_div(s.H, t->MS * t->BH));
  t->tiles_n = s.Cout / t->NT;
  const int64_t tiles = s.N * s.T * t->tiles_h * static_cast<int64_t>(t->tiles_w) * t->tiles_n;
  if (tiles > INT32_MAX) return QVAE_ERR_SHAPE;
  t->num_tiles = static_cast<int>(tiles);
  return QVAE_OK;
}

int check_shape(const qvae_shape* s) {
  if (!s) return QVAE_ERR_ARG;
  if (s->N < 0 || s->T < 0 || s->H < 0 || s->W < 0) return QVAE_ERR_ARG;
  if (s->Cin < 32 || s->Cout < 32 || s->Cin % 32 || s->Cout % 32) return QVAE_ERR_SHAPE;
  const int64_t lim = INT32_MAX / 2;
  if (s->N > lim || s->T > lim || s->H > lim || s->W > lim) return QVAE_ERR_SHAPE;
  // element counts must fit in 63 bits and tensor-map strides in 40 bits
  const double px = static_cast<double>(s->N) * s->T * s->H * s->W;
  if (px * std::max(s->Cin, s->Cout) * 4.0 > 9.0e18) return QVAE_ERR_SHAPE;
  if (static_cast<double>(s->T) * s->H * s->W * s->Cin >= 1099511627776.0) return QVAE_ERR_SHAPE;
  return QVAE_OK;
}

int64_t pixels(const qvae_shape& s) { return s.N * s.T * s.H * s.W; }

int launch_conv(const qvae_shape* shape, const int8_t* xq, const float* x_scale,
                const int8_t* wq, const float* w_scale, const void* bias, void* out, int32_t* acc,
                cudaStream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  const bool acc_mode = acc != nullptr;
  const qvae_shape& s = *shape;
  if (pixels(s) == 0) return QVAE_OK;  // nothing to read or write
  if (!xq || !wq || (!acc_mode && (!x_scale || !w_scale || !out))) return QVAE_ERR_ARG;
  if (!aligned16(xq) || !aligned16(wq) || (out && !aligned16(out)) || (acc && !aligned16(acc)))
    return QVAE_ERR_ALIGN;
  Tiling t;
  rc = make_tiling(s, &t);
  if (rc) return rc;
  int dev;
  rc = current_device(&dev);
  if (rc) return rc;
  int sms;
  rc = sm_count(dev, &sms);
  if (rc) return rc;

  auto encode = tensor_map_encoder();
  if (!encode) {
    t_last_error = "cuTensorMapEncodeTiled is not available from the driver";
    return QVAE_ERR_CUDA;
  }
  CUtensorMap tmap;
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(s.Cin), static_cast<cuuint64_t>(s.W),
                              static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.T),
                              static_cast<cuuint64_t>(s.N)};
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(s.Cin),
                                 static_cast<cuuint64_t>(s.W) * s.Cin,
                                 static_cast<cuuint64_t>(s.H) * s.W * s.Cin,
                                 static_cast<cuuint64_t>(s.T) * s.H * s.W * s.Cin};
  const cuuint32_t box[5] = {128u, static_cast<cuuint32_t>(t.BW),
                             static_cast<cuuint32_t>(t.MS * t.BH + 2), 1u, 1u};
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<int8_t*>(xq), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    char buf[128];
    std::snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(cr));
    t_last_error = buf;
    return QVAE_ERR_CUDA;
  }

  ConvArgs a;
  a.N = static_cast<int>(s.N);
  a.T = static_cast<int>(s.T);
  a.H = static_cast<int>(s.H);
  a.W = static_cast<int>(s.W);
  a.Cin = s.Cin;
  a.Cout = s.Cout;
  a.BW = t.BW;
  a.BH = t.BH;
  a.MS = t.MS;
  a.NT = t.NT;
  a.tiles_w = t.tiles_w;
  a.tiles_h = t.tiles_h;
  a.tiles_n = t.tiles_n;
  a.num_tiles = t.num_tiles;
  a.nchunks = (s.Cin + 127) / 128;
  a.last_ksteps = (s.Cin - (a.nchunks - 1) * 128) / 32;
  a.SA = t.SA;
  a.SB = t.SB;
  a.acc_stages = t.acc_stages;
  a.a_stage_bytes = t.a_stage_bytes;
  a.b_stage_bytes = t.b_stage_bytes;
  a.tmem_cols = t.tmem_cols;
  a.wq = wq;
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.acc_out = acc;
  a.wait_limit_ns = g_wait_limit_ns;

  const int grid = std::min(t.num_tiles, sms);
  if (acc_mode) {
    if (!g_conv_attr_set[dev][1]) {
      QVAE_CUDA(cudaFuncSetAttribute(qvae::conv3d_w8a8_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
      g_conv_attr_set[dev][1] = true;
    }
    qvae::conv3d_w8a8_kernel<true><<<grid, qvae::kConvThreads, t.smem_bytes, stream>>>(tmap, a);
  } else {
    if (!g_conv_attr_set[dev][0]) {
      QVAE_CUDA(cudaFuncSetAttribute(qvae::conv3d_w8a8_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
      g_conv_attr_set[dev][0] = true;
    }
    qvae::conv3d_w8a8_kernel<false><<<grid, qvae::kConvThreads, t.smem_bytes, stream>>>(tmap, a);
  }
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

// ------------------------------------------------------------- activations

int act_grid(int64_t numel, int sms) {
  const int64_t vec = numel / 8;
  const int64_t want = ceil_div(std::max<int64_t>(vec, 1), qvae::kActThreads * 4);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, 4LL * sms)));
}

constexpr size_t kActWorkspace = 16384;  // 4096 partial maxima

int launch_act(const void* x, int64_t numel, int8_t* xq, float* x_scale, void* ws,
               size_t ws_bytes, cudaStream_t stream) {
  if (numel < 0) return QVAE_ERR_ARG;
  if (!x_scale) return QVAE_ERR_ARG;
  if (numel == 0) {
    QVAE_CUDA(cudaMemsetAsync(x_scale, 0, sizeof(float), stream));
    return QVAE_OK;
  }
  if (!x || !xq || !ws) return QVAE_ERR_ARG;
  if (ws_bytes < kActWorkspace) return QVAE_ERR_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(ws)) return QVAE_ERR_ALIGN;
  int dev, sms, rc;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = sm_count(dev, &sms))) return rc;
  const int g1 = act_grid(numel, sms);
  uint32_t* partial = static_cast<uint32_t*>(ws);
  qvae::act_absmax_kernel<<<g1, qvae::kActThreads, 0, stream>>>(
      static_cast<const uint4*>(x), numel / 8, static_cast<const uint16_t*>(x), numel, partial);
  QVAE_CUDA(cudaGetLastError());
  const int64_t nvec2 = numel / 16;
  const int g2 = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(ceil_div(std::max<int64_t>(nvec2, 1), qvae::kActThreads * 2), 4LL * sms)));
  qvae::act_quant_kernel<<<g2, qvae::kActThreads, 0, stream>>>(
      static_cast<const uint4*>(x), nvec2, static_cast<const uint16_t*>(x), numel, partial, g1,
      reinterpret_cast<uint4*>(xq), xq, x_scale);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

// ================================================================== C ABI

extern "C" {

const char* qvae_status_string(int status) {
  switch (status) {
    case QVAE_OK: return "ok";
    case QVAE_ERR_ARG: return "invalid argument";
    case QVAE_ERR_SHAPE: return "unsupported shape (Cin and Cout must be multiples of 32)";
    case QVAE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QVAE_ERR_CUDA: return "CUDA error";
    case QVAE_ERR_TIMEOUT: return "device-side wait timed out";
    case QVAE_ERR_UNSUPPORTED: return "unsupported configuration";
    default: return "unknown status";
  }
}

const char* qvae_last_error_message(void) { return t_last_error.c_str(); }

size_t qvae_packed_weight_bytes(int32_t Cin, int32_t Cout) {
  if (Cin <= 0 || Cout <= 0) return 0;
  return static_cast<size_t>(27) * ((Cin + 127) / 128) * static_cast<size_t>(Cout) * 128;
}

int qvae_quantize_weights(int32_t Cin, int32_t Cout, const void* w_bf16, int8_t* wq_packed,
                          float* w_scale, int8_t* wq_plain, void* stream) {
  if (!w_bf16 || !wq_packed || !w_scale) return QVAE_ERR_ARG;
  if (Cin < 32 || Cout < 32 || Cin % 32 || Cout % 32) return QVAE_ERR_SHAPE;
  if (!aligned16(wq_packed)) return QVAE_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  qvae::weight_scale_kernel<<<Cout, qvae::kWThreads, 0, st>>>(static_cast<const uint16_t*>(w_bf16),
                                                             Cin, w_scale);
  QVAE_CUDA(cudaGetLastError());
  const int nchunks = (Cin + 127) / 128;
  const int64_t total = static_cast<int64_t>(27) * nchunks * Cout * 128;
  const int blocks = static_cast<int>(std::min<int64_t>(ceil_div(total, 256), 65535));
  qvae::weight_pack_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(w_bf16), Cin, Cout,
                                                   nchunks, w_scale, wq_packed, wq_plain);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

size_t qvae_act_workspace_bytes(int64_t numel) {
  (void)numel;
  return kActWorkspace;
}

int qvae_act_absmax_quant(const void* x_bf16, int64_t numel, int8_t* xq, float* x_scale,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return launch_act(x_bf16, numel, xq, x_scale, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream));
}

int qvae_causal_conv3d_w8a8(const qvae_shape* shape, const int8_t* xq, const float* x_scale,
                            const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                            void* out_bf16, void* stream) {
  return launch_conv(shape, xq, x_scale, wq_packed, w_scale, bias_bf16, out_bf16, nullptr,
                     static_cast<cudaStream_t>(stream));
}

int qvae_causal_conv3d_w8a8_acc32(const qvae_shape* shape, const int8_t* xq,
                                  const int8_t* wq_packed, int32_t* acc, void* stream) {
  if (!acc) return QVAE_ERR_ARG;
  return launch_conv(shape, xq, nullptr, wq_packed, nullptr, nullptr, nullptr, acc,
                     static_cast<cudaStream_t>(stream));
}

size_t qvae_decode_workspace_bytes(const qvae_layer* layers, int32_t n) {
  if (!layers || n < 0) return 0;
  int64_t max_in = 0;
  for (int32_t i = 0; i < n; ++i)
    if (layers[i].quantized)
      max_in = std::max<int64_t>(max_in, pixels(layers[i].shape) * layers[i].shape.Cin);
  return align_up(static_cast<size_t>(max_in), 256) + 256 + kActWorkspace;
}

int qvae_decode_layers(const qvae_layer* layers, int32_t n, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (n < 0 || (n > 0 && !layers)) return QVAE_ERR_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const qvae_layer& L = layers[i];
    if (!L.quantized) continue;
    int rc = check_shape(&L.shape);
    if (rc) return rc;
    Tiling t;
    if ((rc = make_tiling(L.shape, &t))) return rc;
    if (!L.x || !L.out || !L.wq_packed || !L.w_scale) return QVAE_ERR_ARG;
    if (!aligned16(L.x) || !aligned16(L.out) || !aligned16(L.wq_packed)) return QVAE_ERR_ALIGN;
  }
  const size_t need = qvae_decode_workspace_bytes(layers, n);
  if (!workspace || workspace_bytes < need) return QVAE_ERR_ARG;
  if (!aligned16(workspace)) return QVAE_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t xq_bytes = need - 256 - kActWorkspace;
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* x_scale = reinterpret_cast<float*>(ws + xq_bytes);
  void* partial = ws + xq_bytes + 256;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t i = 0; i < n; ++i) {
    const qvae_layer& L = layers[i];
    if (!L.quantized) continue;
    const int64_t numel = pixels(L.shape) * L.shape.Cin;
    int rc = launch_act(L.x, numel, xq, x_scale, partial, kActWorkspace, st);
    if (rc) return rc;
    rc = launch_conv(&L.shape, xq, x_scale, L.wq_packed, L.w_scale, L.bias, L.out, nullptr, st);
    if (rc) return rc;
  }
  return QVAE_OK;
}

int qvae_get_error(void* stream) {
  QVAE_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  QVAE_CUDA(cudaMemcpyFromSymbol(&v, qvae::g_qvae_error, sizeof v));
  if (v != 0) {
    const int zero = 0;
    QVAE_CUDA(cudaMemcpyToSymbol(qvae::g_qvae_error, &zero, sizeof zero));
    char buf[64];
    std::snprintf(buf, sizeof buf, "device wait timed out (code 0x%x)", v);
    t_last_error = buf;
    return QVAE_ERR_TIMEOUT;
  }
  return QVAE_OK;
}

int qvae_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns == 0) return QVAE_ERR_ARG;
  g_wait_limit_ns = limit_ns;
  return QVAE_OK;
}

int qvae_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return QVAE_ERR_ARG;
  qvae::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

int qvae_set_conv_tiling(int32_t BW, int32_t MS, int32_t NT, int32_t SA, int32_t SB) {
  if (BW && BW != 8 && BW != 16 && BW != 32 && BW != 64 && BW != 128) return QVAE_ERR_ARG;
  if (MS && MS != 1 && MS != 2) return QVAE_ERR_ARG;
  if (NT && (NT % 32 || NT > 256 || NT < 32)) return QVAE_ERR_ARG;
  if (SA < 0 || SA > qvae::kMaxStages || SB < 0 || SB > qvae::kMaxStages) return QVAE_ERR_ARG;
  g_force[0] = BW;
  g_force[1] = MS;
  g_force[2] = NT;
  g_force[3] = SA;
  g_force[4] = SB;
  return QVAE_OK;
}

int qvae_get_conv_tiling(const qvae_shape* shape, int32_t* out7) {
  if (!out7) return QVAE_ERR_ARG;
  int rc = check_shape(shape);
  if (rc) return rc;
  Tiling t;
  if ((rc = make_tiling(*shape, &t))) return rc;
  out7[0] = t.BW;
  out7[1] = t.BH;
  out7[2] = t.MS;
  out7[3] = t.NT;
  out7[4] = t.SA;
  out7[5] = t.SB;
  out7[6] = t.num_tiles;
  return QVAE_OK;
}

}  // extern "C"
