// qvae.cu -- host side of libqvae: argument checks, tiling choice, tensor-map
// encoding, launches, and the extern "C" entry points declared in qvae.h.
// All kernels live in one translation unit so they share the device error word.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/qvae.h"
#include "conv.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

using qvae::ConvArgs;

thread_local std::string t_last_error;
// Process-wide settings, written by the control entry points and read by every
// launch; atomics so that a setting changed on one host thread while another
// launches is read whole (each value is independent).
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int32_t> g_force[6] = {};   // MS, NT, SA, SB, mode (1 single CTA, 2 CTA pair), G
std::atomic<int32_t> g_cta_limit{0};    // cap on the conv grid (0 = one CTA per SM); tests and tuning

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
bool g_conv_attr_set[kMaxDevices][12] = {};
int g_max_clusters[kMaxDevices][2] = {};  // per device, per thread count (plain, fused)

constexpr int kSmemLimit = 232448;  // dynamic shared memory per block on sm_100

int cuda_fail(cudaError_t e, const char* what) {
  t_last_error = std::string(what) + ": " + cudaGetErrorString(e);
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
  bool pair;
  int MS, NT, SA, SB, acc_stages, G;
  bool split;    // per-sub-tile accumulator hand-off
  int epi_bufs;  // epilogue staging buffers per warp
  bool fuse;     // quantisation in the kernel: a bf16 staging ring of SS row groups
  int SS;
  uint32_t a_stage_bytes, a_box_bytes, b_tap_bytes, b_stage_bytes, tmem_cols, smem_bytes;
  int tiles_w, tiles_h, tiles_n, num_tiles, ctas_per_tile;
  double est_cycles;
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int kStgRows = 2;  // image rows per staging slot of the fused variant (divides 16 * MS + 2)
constexpr uint32_t kStgSlotBytes = kStgRows * qvae::kBoxW * qvae::kStgPixelBytes;

uint32_t smem_needed(const Tiling& t) {
  const uint32_t bars = 8 * qvae::kMaxStages * 4 + 2 * 8 * qvae::kAccBars + 2 * 8 * qvae::kMaxStgSlots + 8;
  return 1024 + t.SA * t.a_stage_bytes + t.SB * t.b_stage_bytes + (t.fuse ? t.SS * kStgSlotBytes : 0u) +
         qvae::kEpiWarps * t.epi_bufs * qvae::kEpiBufBytes +
         bars +
         16 + 16 + 2 * t.NT * 4;
}

// Pipeline depths for a geometry: the deepest weight ring (up to 9 stages of
// G taps each) next to two activation stages and two epilogue staging
// buffers per warp, else the best that fits.  `want_sb`: a weight ring depth
// to reach first with one staging buffer if it does not fit with two (the
// sub-tile hand-off needs a whole chunk's stages).
bool fit_stages_ss(Tiling* t, int want_sb);

bool fit_stages(Tiling* t, int want_sb = 0) {
  if (!t->fuse) {
    t->SS = 0;
    return fit_stages_ss(t, want_sb);
  }
  for (t->SS = 4; t->SS >= 2; t->SS -= 2)
    if (fit_stages_ss(t, want_sb)) return true;
  return false;
}

bool fit_stages_ss(Tiling* t, int want_sb) {
  if (g_force[2] || g_force[3]) {
    t->SA = g_force[2] ? g_force[2].load() : 2;
    t->SB = g_force[3] ? g_force[3].load() : 4;
    for (t->epi_bufs = 2; t->epi_bufs >= 1; --t->epi_bufs)
      if (smem_needed(*t) <= static_cast<uint32_t>(kSmemLimit)) return true;
    return false;
  }
  for (int sa = 2; sa >= 1; --sa) {
    t->SA = sa;
    for (int bufs = 2; bufs >= 1; --bufs) {
      t->epi_bufs = bufs;
      for (t->SB = 9; t->SB >= 2; --t->SB) {
        if (smem_needed(*t) > static_cast<uint32_t>(kSmemLimit)) continue;
        if (bufs == 2 && want_sb && t->SB < want_sb) break;  // try one staging buffer
        return true;
      }
    }
  }
  return false;
}

// Relative cost of a geometry on `sms` SMs, in SM cycles: waves x the time of
// a CTA tile.  A tile is its weight stages (G taps of one 128-channel chunk
// each), each tap MS x k-steps MMAs of 128 x NT x 32 at the measured cycles
// per MMA for that N, plus a handshake per stage, an exposed activation load
// per chunk when the activation ring has one stage, and the epilogue time an
// accumulator buffer leaves exposed: none with two buffers (the next tile's
// MMAs run beside it) except the last tile's; one sub-tile's with a single
// buffer handed over sub-tile by sub-tile; all sub-tiles' otherwise.  The
// exposed epilogue measured about 16 cycles per accumulator column and
// sub-tile (the term that makes one sub-tile with two buffers beat two
// sub-tiles with one on the 192-channel layers, as measured).  A CTA pair's
// MMAs are issued once for both SMs and each SM loads half the weights: pairs
// measured 25-40 % faster than single CTAs of the same geometry (the MMA
// issue, not the tensor pipe, bounds the narrow layers).
double estimate_cycles(const qvae_shape& s, const Tiling& t, int sms) {
  double taps_t = 0;
  for (int64_t f = 0; f < std::min<int64_t>(s.T, 2); ++f) taps_t += static_cast<double>(f + 1);
  if (s.T > 2) taps_t += 3.0 * (s.T - 2);
  taps_t /= s.T;
  // cycles per MMA measured with random data: N=96 86, 128 91, 192 109, 256 143
  const double mma = std::max(0.52 * t.NT + 8.0, 60.0 + 0.17 * t.NT);
  constexpr double kEpi = 16.0;  // exposed epilogue cycles per accumulator column and sub-tile
  const int nchunks = (s.Cin + 127) / 128;
  const double ksteps_total = s.Cin / 32.0;
  const double stages = taps_t * 9.0 / t.G * nchunks;
  const double exposed = t.acc_stages == 2 ? 0.0 : kEpi * (t.split ? 1 : t.MS) * t.NT;
  const double per_tile = taps_t * 9.0 * ksteps_total * t.MS * mma + stages * 250.0 + 500.0 +
                          (t.SA == 1 ? 1500.0 * taps_t * nchunks : 0.0) + exposed;
  const double slots = t.pair ? std::floor(sms / 2.0) : sms;
  const double waves = std::ceil(static_cast<double>(t.num_tiles) / slots);
  // the last tile's epilogue (its last sub-tile's when they are handed over one by one)
  const double tail = t.acc_stages == 2 ? kEpi * t.MS * t.NT : (t.split ? kEpi * t.NT : 0.0);
  return (waves * per_tile + tail) * (t.pair ? 1.0 : 1.3);
}

int make_geometry(const qvae_shape& s, bool pair, int MS, int NT, int G, int sms, Tiling* t, bool fuse) {
  if (G != 1 && !(G == 3 && MS <= 2)) return QVAE_ERR_ARG;  // kernel instantiations
  t->fuse = fuse;
  t->pair = pair;
  t->MS = MS;
  t->NT = NT;
  t->G = G;
  t->ctas_per_tile = pair ? 2 : 1;
  const int rows = MS * qvae::kTileRows + 2;
  t->a_box_bytes = static_cast<uint32_t>(rows) * qvae::kGroupStride;
  t->a_stage_bytes = (t->a_box_bytes + 1023u) & ~1023u;
  t->b_tap_bytes = static_cast<uint32_t>(pair ? NT / 2 : NT) * 128u;
  t->b_stage_bytes = static_cast<uint32_t>(G) * t->b_tap_bytes;
  const int acc_cols = MS * NT;
  if (acc_cols > 512) return QVAE_ERR_ARG;
  t->acc_stages = (2 * acc_cols <= 512) ? 2 : 1;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(t->acc_stages * acc_cols)) cols <<= 1;
  t->tmem_cols = cols;
  t->tiles_w = static_cast<int>(ceil_div(s.W, qvae::kTileW));
  t->tiles_h = static_cast<int>(ceil_div(s.H, MS * qvae::kTileRows * t->ctas_per_tile));
  t->tiles_n = s.Cout / NT;
  const int64_t tiles = s.N * s.T * t->tiles_h * static_cast<int64_t>(t->tiles_w) * t->tiles_n;
  if (tiles > INT32_MAX / 2) return QVAE_ERR_SHAPE;
  t->num_tiles = static_cast<int>(tiles);
  // One accumulator buffer of several sub-tiles: hand them over one by one
  // when the weight ring holds a whole chunk's stages.  The hand-off pays
  // when CTAs walk several tiles; with about one tile per CTA two staging
  // buffers per epilogue warp (a faster last epilogue) measured better.
  const int slots = pair ? std::max(1, sms / 2) : std::max(1, sms);
  const bool want_split = t->acc_stages == 1 && MS >= 2 && 2 * t->num_tiles >= 3 * slots;
  if (!fit_stages(t, want_split ? 9 / G : 0)) return QVAE_ERR_UNSUPPORTED;
  t->smem_bytes = smem_needed(*t);
  t->split = t->acc_stages == 1 && MS >= 2 && t->SB >= 9 / G;
  return QVAE_OK;
}

int make_tiling(const qvae_shape& s, Tiling* t, int sms = 148, bool fuse = false) {
  bool found = false;
  for (int mode = 1; mode <= 2; ++mode) {
    if (g_force[4] && mode != g_force[4]) continue;
    for (int ms = 1; ms <= 4; ++ms) {
      if (g_force[0] && ms != g_force[0]) continue;
      for (int nt = 32; nt <= std::min(256, s.Cout); nt += 32) {
        if (s.Cout % nt) continue;
        if (g_force[1] && nt != g_force[1]) continue;
        for (int g = 1; g <= 3; g += 2) {
          if (g_force[5] && g != g_force[5]) continue;
          Tiling u;
          if (make_geometry(s, mode == 2, ms, nt, g, sms, &u, fuse) != QVAE_OK) continue;
          u.est_cycles = estimate_cycles(s, u, sms);
          if (!found || u.est_cycles < t->est_cycles) {
            *t = u;
            found = true;
          }
        }
      }
    }
  }
  return found ? QVAE_OK : QVAE_ERR_UNSUPPORTED;
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

int encode_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, const cuuint64_t* dims,
               const cuuint64_t* strides, const cuuint32_t* box, int rank, CUtensorMapSwizzle swizzle) {
  auto encode = tensor_map_encoder();
  if (!encode) {
    t_last_error = "cuTensorMapEncodeTiled is not available from the driver";
    return QVAE_ERR_CUDA;
  }
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult cr = encode(map, dtype, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    char buf[128];
    std::snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(cr));
    t_last_error = buf;
    return QVAE_ERR_CUDA;
  }
  return QVAE_OK;
}

// Launch as a programmatic dependent of the previous kernel on the stream:
// the grid may start while its predecessor finishes and synchronises with
// griddepcontrol.wait before touching the predecessor's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                             cudaStream_t stream, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// carry: xq holds T + 2 frames per batch item, the first two carried from
// the previous chunk of a streamed video (output frames are the last T).
// halo_top / halo_bot: xq holds H + halo_top + halo_bot rows, output row h
// reading input rows h + halo_top - 1 .. h + halo_top + 1 (a row band).
// bf16: the native-precision convolution -- xq holds bf16 values, wq the bf16
// packing, acc (accumulator mode) receives fp32 sums; no scales.  It is tiled
// as the INT8 convolution of twice the channels (the same bytes per pixel).
// x_amax != null: the fused W8A8 variant -- xq holds the bf16 input, quantised
// in the kernel with the scale bf16(*x_amax) / 127; x_scale_out (nullable)
// receives that scale; zero_word (nullable) is set to zero by the kernel.
int launch_conv(const qvae_shape* shape, const void* xq, const float* x_scale,
                const void* wq, const float* w_scale, const void* bias, void* out, void* acc,
                cudaStream_t stream, bool carry = false, uint32_t* out_amax = nullptr, int halo_top = 0,
                int halo_bot = 0, bool bf16 = false, const uint32_t* x_amax = nullptr,
                float* x_scale_out = nullptr, uint32_t* zero_word = nullptr) {
  int rc = check_shape(shape);
  if (rc) return rc;
  const bool fuse = x_amax != nullptr;
  if (fuse && bf16) return QVAE_ERR_ARG;
  const int elt = bf16 ? 2 : 1;            // bytes per operand element in shared memory
  const int x_elt = (bf16 || fuse) ? 2 : 1;  // bytes per input element in global memory
  if (halo_top < 0 || halo_top > 1 || halo_bot < 0 || halo_bot > 1) return QVAE_ERR_ARG;
  // the input tensor map's largest stride (one batch item) must fit 40 bits
  if (static_cast<double>(shape->T + (carry ? 2 : 0)) * (shape->H + halo_top + halo_bot) * shape->W *
          shape->Cin * x_elt >= 1099511627776.0)
    return QVAE_ERR_SHAPE;
  const bool acc_mode = acc != nullptr;
  const qvae_shape& s = *shape;
  if (pixels(s) == 0) return QVAE_OK;  // nothing to read or write
  if (!xq || !wq || (!acc_mode && !out) || (!acc_mode && !bf16 && ((!x_scale && !fuse) || !w_scale)))
    return QVAE_ERR_ARG;
  if (!aligned16(xq) || !aligned16(wq) || (out && !aligned16(out)) || (acc && !aligned16(acc)))
    return QVAE_ERR_ALIGN;
  int dev;
  rc = current_device(&dev);
  if (rc) return rc;
  int sms;
  rc = sm_count(dev, &sms);
  if (rc) return rc;
  qvae_shape sb = s;  // the geometry in bytes: bf16 is tiled as twice the channels of codes
  sb.Cin = s.Cin * elt;
  Tiling t;
  rc = make_tiling(sb, &t, sms, fuse);
  if (rc) return rc;
  const int nchunks = (sb.Cin + 127) / 128;  // 128-byte channel chunks

  CUtensorMap tmap_x, tmap_w, tmap_out;
  {
    const cuuint64_t t_in = static_cast<cuuint64_t>(s.T) + (carry ? 2 : 0);
    const cuuint64_t h_in = static_cast<cuuint64_t>(s.H) + halo_top + halo_bot;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(s.Cin), static_cast<cuuint64_t>(s.W), h_in, t_in,
                                static_cast<cuuint64_t>(s.N)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(s.Cin) * x_elt,
                                   static_cast<cuuint64_t>(s.W) * s.Cin * x_elt,
                                   h_in * s.W * s.Cin * x_elt,
                                   t_in * h_in * s.W * s.Cin * x_elt};
    if (fuse) {
      // bf16 row groups of the box for the staging ring: 128 channels x 10 columns x kStgRows rows
      const cuuint32_t box[5] = {128u, static_cast<cuuint32_t>(qvae::kBoxW), static_cast<cuuint32_t>(kStgRows), 1u, 1u};
      rc = encode_map(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xq, dims, strides, box, 5,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
      const cuuint32_t box[5] = {128u / elt, static_cast<cuuint32_t>(qvae::kBoxW),
                                 static_cast<cuuint32_t>(t.MS * qvae::kTileRows + 2), 1u, 1u};
      rc = encode_map(&tmap_x, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, dims,
                      strides, box, 5, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (rc) return rc;
  }
  {
    // packed weights as rows of 128 bytes: [tap][chunk][Cout] rows
    const cuuint64_t dims[2] = {128u, static_cast<cuuint64_t>(27) * nchunks * s.Cout};
    const cuuint64_t strides[1] = {128u};
    const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(t.pair ? t.NT / 2 : t.NT)};
    rc = encode_map(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, dims, strides, box, 2,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  if (!acc_mode) {
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(s.Cout), static_cast<cuuint64_t>(s.W),
                                static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.T),
                                static_cast<cuuint64_t>(s.N)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(s.Cout) * 2,
                                   static_cast<cuuint64_t>(s.W) * s.Cout * 2,
                                   static_cast<cuuint64_t>(s.H) * s.W * s.Cout * 2,
                                   static_cast<cuuint64_t>(s.T) * s.H * s.W * s.Cout * 2};
    // one epilogue warp's slice: 32 channels x 8 columns x 4 rows
    const cuuint32_t box[5] = {32u, static_cast<cuuint32_t>(qvae::kTileW), 4u, 1u, 1u};
    rc = encode_map(&tmap_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, dims, strides, box, 5,
                    CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
  } else {
    tmap_out = tmap_x;  // unused by the accumulator variant
  }

  ConvArgs a;
  a.N = static_cast<int>(s.N);
  a.T = static_cast<int>(s.T);
  a.H = static_cast<int>(s.H);
  a.W = static_cast<int>(s.W);
  a.Cin = s.Cin;
  a.Cout = s.Cout;
  a.MS = t.MS;
  a.NT = t.NT;
  a.tiles_w = t.tiles_w;
  a.tiles_h = t.tiles_h;
  a.tiles_n = t.tiles_n;
  a.num_tiles = t.num_tiles;
  a.nchunks = nchunks;
  a.last_ksteps = (sb.Cin - (nchunks - 1) * 128) / 32;
  a.chunk_elems = 128 / elt;
  a.SA = t.SA;
  a.SB = t.SB;
  a.acc_stages = t.acc_stages;
  a.a_stage_bytes = t.a_stage_bytes;
  a.a_box_bytes = t.a_box_bytes;
  a.G = t.G;
  a.split = t.split ? 1 : 0;
  a.epi_bufs = t.epi_bufs;
  a.carry = carry ? 1 : 0;
  a.halo_top = halo_top;
  a.out_amax = acc_mode ? nullptr : out_amax;
  a.b_tap_bytes = t.b_tap_bytes;
  a.b_stage_bytes = t.b_stage_bytes;
  a.tmem_cols = t.tmem_cols;
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.acc_out = static_cast<int32_t*>(acc);
  a.wait_limit_ns = g_wait_limit_ns;
  a.x_amax = x_amax;
  a.x_scale_out = x_scale_out;
  a.zero_word = zero_word;
  a.one = 1.0f;
  a.SS = t.SS;
  a.stg_rows = kStgRows;
  a.stg_groups = (t.MS * qvae::kTileRows + 2) / kStgRows;
  a.stg_slot_bytes = kStgSlotBytes;

  const int kidx = (acc_mode ? 1 : 0) + (t.pair ? 2 : 0) + (bf16 ? 4 : 0) + (fuse ? 8 : 0);
  using Kernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, qvae::ConvArgs);
  const Kernel kernels[12] = {
      qvae::conv3d_w8a8_kernel<false, false>,       qvae::conv3d_w8a8_kernel<true, false>,
      qvae::conv3d_w8a8_kernel<false, true>,        qvae::conv3d_w8a8_kernel<true, true>,
      qvae::conv3d_bf16_kernel<false, false>,       qvae::conv3d_bf16_kernel<true, false>,
      qvae::conv3d_bf16_kernel<false, true>,        qvae::conv3d_bf16_kernel<true, true>,
      qvae::conv3d_w8a8_fused_kernel<false, false>, qvae::conv3d_w8a8_fused_kernel<true, false>,
      qvae::conv3d_w8a8_fused_kernel<false, true>,  qvae::conv3d_w8a8_fused_kernel<true, true>};
  const int threads = fuse ? qvae::kConvThreadsFused : qvae::kConvThreads;
  const Kernel kernel = kernels[kidx];
  if (!g_conv_attr_set[dev][kidx]) {
    QVAE_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    g_conv_attr_set[dev][kidx] = true;
  }
  int grid;
  if (t.pair) {
    int& max_clusters = g_max_clusters[dev][fuse ? 1 : 0];
    if (max_clusters == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * sms);
      cfg.blockDim = dim3(threads);
      cfg.dynamicSmemBytes = kSmemLimit;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      QVAE_CUDA(cudaOccupancyMaxActiveClusters(&n, kernel, &cfg));
      max_clusters = std::max(n, 1);
    }
    const int cta_limit = g_cta_limit.load();
    int clusters = std::min(t.num_tiles, max_clusters);
    if (cta_limit > 0) clusters = std::max(1, std::min(clusters, cta_limit / 2));
    grid = 2 * clusters;
  } else {
    const int cta_limit = g_cta_limit.load();
    grid = std::min(t.num_tiles, sms);
    if (cta_limit > 0) grid = std::min(grid, cta_limit);
  }
  QVAE_CUDA(launch_dependent(kernel, grid, threads, t.smem_bytes, stream, t.pair ? 2 : 1, tmap_x,
                             tmap_w, tmap_out, a));
  return QVAE_OK;
}

// ------------------------------------------------------------- activations

// Blocks of the absmax pass: enough for kAbsUnroll vectors per thread, at
// most kActBlocksPerSm 256-thread blocks per SM (full occupancy).
constexpr int kActBlocksPerSm = 8;
int act_grid(int64_t numel, int sms) {
  const int64_t vec = numel / 8;
  const int64_t want = ceil_div(std::max<int64_t>(vec, 1), qvae::kActThreads * qvae::kAbsUnroll);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(kActBlocksPerSm) * sms)));
}

// Blocks of the quantise pass: kQuantUnroll 16-value groups per thread, at
// most eight blocks per SM.
int quant_grid(int64_t numel, int sms) {
  const int64_t nvec2 = numel / 16;
  const int64_t want = ceil_div(std::max<int64_t>(nvec2, 1), qvae::kActThreads * qvae::kQuantUnroll);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(kActBlocksPerSm) * sms)));
}

constexpr size_t kActWorkspace = 16384;  // 4096 partial maxima: enough for 512 SMs

// zero_word (nullable): a device word the quantise pass sets to zero, for a
// following convolution to accumulate its output maximum into.
int launch_act(const void* x, int64_t numel, int8_t* xq, float* x_scale, void* ws,
               size_t ws_bytes, cudaStream_t stream, uint32_t* zero_word = nullptr) {
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
  if (static_cast<size_t>(g1) * sizeof(uint32_t) > ws_bytes) {
    t_last_error = "the activation workspace holds fewer partial maxima than this GPU's absmax pass writes";
    return QVAE_ERR_UNSUPPORTED;
  }
  uint32_t* partial = static_cast<uint32_t*>(ws);
  qvae::act_absmax_kernel<<<g1, qvae::kActThreads, 0, stream>>>(
      static_cast<const uint4*>(x), numel / 8, static_cast<const uint16_t*>(x), numel, partial, nullptr);
  QVAE_CUDA(cudaGetLastError());
  const int64_t nvec2 = numel / 16;
  const int g2 = quant_grid(numel, sms);
  QVAE_CUDA(launch_dependent(qvae::act_quant_kernel, g2, qvae::kActThreads, 0, stream, 1,
                             static_cast<const uint4*>(x), nvec2, static_cast<const uint16_t*>(x), numel,
                             static_cast<const uint32_t*>(partial), g1, reinterpret_cast<uint4*>(xq), xq,
                             x_scale, zero_word));
  return QVAE_OK;
}

// The quantise pass alone, for an input whose absmax (15-bit bf16 magnitude)
// the previous convolution accumulated into *amax while writing it.  A plain
// launch: the input is that convolution's output, so nothing of this kernel
// may run before it has finished.
int launch_quant_from_amax(const void* x, int64_t numel, const uint32_t* amax, int8_t* xq, float* x_scale,
                           uint32_t* zero_word, cudaStream_t stream) {
  if (numel == 0) {
    QVAE_CUDA(cudaMemsetAsync(x_scale, 0, sizeof(float), stream));
    return QVAE_OK;
  }
  int dev, sms, rc;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = sm_count(dev, &sms))) return rc;
  const int64_t nvec2 = numel / 16;
  const int g2 = quant_grid(numel, sms);
  qvae::act_quant_kernel<<<g2, qvae::kActThreads, 0, stream>>>(
      static_cast<const uint4*>(x), nvec2, static_cast<const uint16_t*>(x), numel, amax, 1,
      reinterpret_cast<uint4*>(xq), xq, x_scale, zero_word);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

}  // namespace

// ====================================================== fixed device scratch
// For callers that cannot allocate device memory, qvae_act_absmax_quant_noalloc
// keeps the activation quantiser's partial maxima in this fixed array instead
// of a caller workspace.  Every GPU that loads the library holds it (16 KiB)
// until the process exits.
namespace {

constexpr int kStaticPartialSlots = 4096;  // one 32-bit partial maximum per absmax CTA (512 SMs x 8)
static __device__ __align__(256) uint32_t g_static_partials[kStaticPartialSlots];

void* g_static_partials_addr[kMaxDevices] = {};
std::mutex g_static_mutex;

// The device address of the array on the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up once per
// device (with that device current) and cached.
int static_partials(int dev, uint32_t** out) {
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_partials_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_partials);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static partial maxima)");
    g_static_partials_addr[dev] = p;
  }
  *out = static_cast<uint32_t*>(g_static_partials_addr[dev]);
  return QVAE_OK;
}

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
    case QVAE_ERR_BOUNDS: return "a device bounds check failed (debug build)";
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
  qvae::stream_fence_kernel<<<1, 32, 0, st>>>();  // see the convolution's early weight loads
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

int qvae_act_absmax(const void* x_bf16, int64_t numel, uint32_t* amax, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (numel < 0 || !amax) return QVAE_ERR_ARG;
  if (numel > 0 && !x_bf16) return QVAE_ERR_ARG;
  if (numel > 0 && !aligned16(x_bf16)) return QVAE_ERR_ALIGN;
  QVAE_CUDA(cudaMemsetAsync(amax, 0, sizeof(uint32_t), st));
  if (numel == 0) return QVAE_OK;
  int dev, sms, rc;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = sm_count(dev, &sms))) return rc;
  qvae::act_absmax_kernel<<<act_grid(numel, sms), qvae::kActThreads, 0, st>>>(
      static_cast<const uint4*>(x_bf16), numel / 8, static_cast<const uint16_t*>(x_bf16), numel, nullptr,
      amax);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

int qvae_act_quant_from_absmax(const void* x_bf16, int64_t numel, const uint32_t* amax, int8_t* xq,
                               float* x_scale, void* stream) {
  if (numel < 0 || !amax || !x_scale) return QVAE_ERR_ARG;
  if (numel > 0 && (!x_bf16 || !xq)) return QVAE_ERR_ARG;
  if (numel > 0 && (!aligned16(x_bf16) || !aligned16(xq))) return QVAE_ERR_ALIGN;
  return launch_quant_from_amax(x_bf16, numel, amax, xq, x_scale, nullptr, static_cast<cudaStream_t>(stream));
}

int qvae_causal_conv3d_w8a8_band(const qvae_shape* shape, int32_t halo_top, int32_t halo_bot,
                                 const int8_t* xq_band, const float* x_scale, const int8_t* wq_packed,
                                 const float* w_scale, const void* bias_bf16, void* out_bf16, void* stream) {
  return launch_conv(shape, xq_band, x_scale, wq_packed, w_scale, bias_bf16, out_bf16, nullptr,
                     static_cast<cudaStream_t>(stream), false, nullptr, halo_top, halo_bot);
}

int qvae_causal_conv3d_w8a8_band_acc32(const qvae_shape* shape, int32_t halo_top, int32_t halo_bot,
                                       const int8_t* xq_band, const int8_t* wq_packed, int32_t* acc,
                                       void* stream) {
  if (!acc) return QVAE_ERR_ARG;
  return launch_conv(shape, xq_band, nullptr, wq_packed, nullptr, nullptr, nullptr, acc,
                     static_cast<cudaStream_t>(stream), false, nullptr, halo_top, halo_bot);
}

int qvae_causal_conv3d_w8a8_carry(const qvae_shape* shape, const int8_t* xq_ext, const float* x_scale,
                                  const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                                  void* out_bf16, void* stream) {
  return launch_conv(shape, xq_ext, x_scale, wq_packed, w_scale, bias_bf16, out_bf16, nullptr,
                     static_cast<cudaStream_t>(stream), true);
}

int qvae_causal_conv3d_w8a8_carry_acc32(const qvae_shape* shape, const int8_t* xq_ext,
                                        const int8_t* wq_packed, int32_t* acc, void* stream) {
  if (!acc) return QVAE_ERR_ARG;
  return launch_conv(shape, xq_ext, nullptr, wq_packed, nullptr, nullptr, nullptr, acc,
                     static_cast<cudaStream_t>(stream), true);
}

size_t qvae_packed_weight_bytes_bf16(int32_t Cin, int32_t Cout) {
  if (Cin <= 0 || Cout <= 0) return 0;
  return static_cast<size_t>(27) * ((Cin + 63) / 64) * static_cast<size_t>(Cout) * 128;
}

int qvae_pack_weights_bf16(int32_t Cin, int32_t Cout, const void* w_bf16, void* w_packed, void* stream) {
  if (!w_bf16 || !w_packed) return QVAE_ERR_ARG;
  if (Cin < 32 || Cout < 32 || Cin % 32 || Cout % 32) return QVAE_ERR_SHAPE;
  if (!aligned16(w_packed)) return QVAE_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nchunks = (Cin + 63) / 64;
  const int64_t total = static_cast<int64_t>(27) * nchunks * Cout * 64;
  const int blocks = static_cast<int>(std::min<int64_t>(ceil_div(total, 256), 65535));
  qvae::weight_pack_bf16_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(w_bf16), Cin, Cout, nchunks,
                                                        static_cast<uint16_t*>(w_packed));
  QVAE_CUDA(cudaGetLastError());
  qvae::stream_fence_kernel<<<1, 32, 0, st>>>();  // see the convolution's early weight loads
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

int qvae_causal_conv3d_bf16(const qvae_shape* shape, const void* x_bf16, const void* w_packed,
                            const void* bias_bf16, void* out_bf16, void* stream) {
  return launch_conv(shape, x_bf16, nullptr, w_packed, nullptr, bias_bf16, out_bf16, nullptr,
                     static_cast<cudaStream_t>(stream), false, nullptr, 0, 0, true);
}

int qvae_causal_conv3d_bf16_acc32(const qvae_shape* shape, const void* x_bf16, const void* w_packed,
                                  float* acc, void* stream) {
  if (!acc) return QVAE_ERR_ARG;
  return launch_conv(shape, x_bf16, nullptr, w_packed, nullptr, nullptr, nullptr, acc,
                     static_cast<cudaStream_t>(stream), false, nullptr, 0, 0, true);
}

int qvae_causal_conv3d_w8a8_fused(const qvae_shape* shape, const void* x_bf16, const uint32_t* x_amax,
                                  const int8_t* wq_packed, const float* w_scale, const void* bias_bf16,
                                  void* out_bf16, float* x_scale_out, void* stream) {
  if (!x_amax) return QVAE_ERR_ARG;
  return launch_conv(shape, x_bf16, nullptr, wq_packed, w_scale, bias_bf16, out_bf16, nullptr,
                     static_cast<cudaStream_t>(stream), false, nullptr, 0, 0, false, x_amax, x_scale_out);
}

int qvae_causal_conv3d_w8a8_fused_acc32(const qvae_shape* shape, const void* x_bf16, const uint32_t* x_amax,
                                        const int8_t* wq_packed, int32_t* acc, void* stream) {
  if (!x_amax || !acc) return QVAE_ERR_ARG;
  return launch_conv(shape, x_bf16, nullptr, wq_packed, nullptr, nullptr, nullptr, acc,
                     static_cast<cudaStream_t>(stream), false, nullptr, 0, 0, false, x_amax);
}

int qvae_act_absmax_quant_noalloc(const void* x_bf16, int64_t numel, int8_t* xq, float* x_scale,
                                  void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (numel < 0 || !x_scale) return QVAE_ERR_ARG;
  if (numel == 0) {
    QVAE_CUDA(cudaMemsetAsync(x_scale, 0, sizeof(float), st));
    return QVAE_OK;
  }
  if (!x_bf16 || !xq) return QVAE_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(xq)) return QVAE_ERR_ALIGN;
  int dev, sms, rc;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = sm_count(dev, &sms))) return rc;
  const int g1 = act_grid(numel, sms);
  if (g1 > kStaticPartialSlots) {
    char buf[160];
    std::snprintf(buf, sizeof buf,
                  "this launch needs %d partial-maximum slots; the fixed scratch holds %d", g1,
                  kStaticPartialSlots);
    t_last_error = buf;
    return QVAE_ERR_UNSUPPORTED;
  }
  uint32_t* partial = nullptr;
  if ((rc = static_partials(dev, &partial))) return rc;
  // Same two kernels as qvae_act_absmax_quant; every slot the second reads is
  // written by the first in this call, so nothing needs clearing.
  qvae::act_absmax_kernel<<<g1, qvae::kActThreads, 0, st>>>(
      static_cast<const uint4*>(x_bf16), numel / 8, static_cast<const uint16_t*>(x_bf16), numel, partial,
      nullptr);
  QVAE_CUDA(cudaGetLastError());
  const int64_t nvec2 = numel / 16;
  const int g2 = quant_grid(numel, sms);
  QVAE_CUDA(launch_dependent(qvae::act_quant_kernel, g2, qvae::kActThreads, 0, st, 1,
                             static_cast<const uint4*>(x_bf16), nvec2, static_cast<const uint16_t*>(x_bf16),
                             numel, static_cast<const uint32_t*>(partial), g1, reinterpret_cast<uint4*>(xq), xq,
                             x_scale, static_cast<uint32_t*>(nullptr)));
  return QVAE_OK;
}

// Workspace of qvae_decode_layers: the activation scale of the last quantised
// layer (fp32 at byte 0) and three 32-bit maximum words (bytes 64, 128, 192);
// then, when quantised layers run as the quantise pass + the convolution of
// codes, the activation workspace (partial maxima) and the largest quantised
// input's codes.
constexpr size_t kDecodeHeader = 256;

std::atomic<bool> g_fused_quant{false};  // quantised layers of qvae_decode_layers: fused convolution

size_t qvae_decode_workspace_bytes(const qvae_layer* layers, int32_t n) {
  if (!layers || n < 0) return 0;
  if (g_fused_quant) return kDecodeHeader;
  int64_t max_in = 0;
  for (int32_t i = 0; i < n; ++i)
    if (layers[i].quantized) max_in = std::max<int64_t>(max_in, pixels(layers[i].shape) * layers[i].shape.Cin);
  return kDecodeHeader + kActWorkspace + static_cast<size_t>((max_in + 255) / 256 * 256);
}

// The library runs a layer when it is quantised, or when it is a native-
// precision layer given bf16 weights packed by qvae_pack_weights_bf16.
bool runs(const qvae_layer& L) { return L.quantized || L.wq_packed; }

// Layer i's output is, element for element, layer i + 1's input and layer
// i + 1 is quantised (same pixels, Cout == next Cin, same pointer): layer i's
// epilogue can take the maximum that layer i + 1's quantiser needs.
bool feeds_next(const qvae_layer* layers, int32_t n, int32_t i) {
  if (i + 1 >= n) return false;
  const qvae_layer &a = layers[i], &b = layers[i + 1];
  return runs(a) && b.quantized && a.out == b.x && a.shape.N == b.shape.N && a.shape.T == b.shape.T &&
         a.shape.H == b.shape.H && a.shape.W == b.shape.W && a.shape.Cout == b.shape.Cin;
}

int qvae_decode_layers(const qvae_layer* layers, int32_t n, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (n < 0 || (n > 0 && !layers)) return QVAE_ERR_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const qvae_layer& L = layers[i];
    if (!runs(L)) continue;
    int rc = check_shape(&L.shape);
    if (rc) return rc;
    if (!L.x || !L.out || !L.wq_packed || (L.quantized && !L.w_scale)) return QVAE_ERR_ARG;
    if (!aligned16(L.x) || !aligned16(L.out) || !aligned16(L.wq_packed)) return QVAE_ERR_ALIGN;
  }
  const size_t need = qvae_decode_workspace_bytes(layers, n);
  if (!workspace || workspace_bytes < need) return QVAE_ERR_ARG;
  if (!aligned16(workspace)) return QVAE_ERR_ALIGN;
  if (n > 0) {
    // every shape has a valid tiling on this GPU before anything is launched
    int dev = 0, sms = 0, rc = current_device(&dev);
    if (rc) return rc;
    if ((rc = sm_count(dev, &sms))) return rc;
    for (int32_t i = 0; i < n; ++i) {
      if (!runs(layers[i])) continue;
      qvae_shape sb = layers[i].shape;
      if (!layers[i].quantized) sb.Cin *= 2;  // a native layer is tiled by bytes
      Tiling t;
      if ((rc = make_tiling(sb, &t, sms, layers[i].quantized != 0 && g_fused_quant))) return rc;
    }
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* x_scale = reinterpret_cast<float*>(ws);
  const bool fused = g_fused_quant.load();
  void* partial = ws + kDecodeHeader;
  int8_t* xq = reinterpret_cast<int8_t*>(ws + kDecodeHeader + kActWorkspace);
  // Layer i reads its input maximum from word i % 3, accumulates its output's
  // maximum (when that output feeds the next quantised layer) into word
  // (i + 1) % 3, and a fused convolution clears word (i + 2) % 3: the word
  // layer i + 1 will accumulate into, which nothing reads or writes from the
  // moment layer i starts (layer i - 1, its last reader, has finished).
  uint32_t* word[3] = {reinterpret_cast<uint32_t*>(ws + 64), reinterpret_cast<uint32_t*>(ws + 128),
                       reinterpret_cast<uint32_t*>(ws + 192)};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n > 0) QVAE_CUDA(cudaMemsetAsync(ws + 64, 0, 192, st));
  bool next_cleared = true;  // the word this layer accumulates into is zero
  for (int32_t i = 0; i < n; ++i) {
    const qvae_layer& L = layers[i];
    if (!runs(L)) {
      next_cleared = false;
      continue;
    }
    const bool feeds = feeds_next(layers, n, i);
    uint32_t* in_word = word[i % 3];
    uint32_t* out_word = feeds ? word[(i + 1) % 3] : nullptr;
    // the quantise pass of the two-pass path clears out_word itself
    if (out_word && !next_cleared && (fused || !L.quantized))
      QVAE_CUDA(cudaMemsetAsync(out_word, 0, sizeof(uint32_t), st));
    int rc;
    if (!L.quantized) {
      // native precision: the bf16 convolution straight from the bf16 input
      rc = launch_conv(&L.shape, L.x, nullptr, L.wq_packed, nullptr, L.bias, L.out, nullptr, st, false, out_word,
                       0, 0, true);
      next_cleared = false;
    } else {
      const bool fed = i > 0 && feeds_next(layers, n, i - 1);  // input maximum already accumulated
      const int64_t numel = pixels(L.shape) * L.shape.Cin;
      if (fused) {
        if (!fed && (rc = qvae_act_absmax(L.x, numel, in_word, st))) return rc;
        rc = launch_conv(&L.shape, L.x, nullptr, L.wq_packed, L.w_scale, L.bias, L.out, nullptr, st, false,
                         out_word, 0, 0, false, in_word, x_scale, word[(i + 2) % 3]);
        next_cleared = true;
      } else {
        // quantise pass (which also clears out_word), then the convolution of the codes
        rc = fed ? launch_quant_from_amax(L.x, numel, in_word, xq, x_scale, out_word, st)
                 : launch_act(L.x, numel, xq, x_scale, partial, kActWorkspace, st, out_word);
        if (rc) return rc;
        rc = launch_conv(&L.shape, xq, x_scale, L.wq_packed, L.w_scale, L.bias, L.out, nullptr, st, false,
                         out_word);
        next_cleared = false;
      }
    }
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
    if (v == qvae::kErrBounds) {
      std::snprintf(buf, sizeof buf, "device bounds check failed (code 0x%x)", v);
      t_last_error = buf;
      return QVAE_ERR_BOUNDS;
    }
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

int qvae_build_flags(void) {
#ifdef QVAE_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

int qvae_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return QVAE_ERR_ARG;
  qvae::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  QVAE_CUDA(cudaGetLastError());
  return QVAE_OK;
}

int qvae_set_conv_tiling(int32_t MS, int32_t NT, int32_t SA, int32_t SB, int32_t mode, int32_t G) {
  if (MS < 0 || MS > 4) return QVAE_ERR_ARG;
  if (NT && (NT % 32 || NT > 256 || NT < 32)) return QVAE_ERR_ARG;
  if (MS && NT && MS * NT > 512) return QVAE_ERR_ARG;
  if (SA < 0 || SA > qvae::kMaxStages || SB < 0 || SB > qvae::kMaxStages) return QVAE_ERR_ARG;
  if (mode < 0 || mode > 2) return QVAE_ERR_ARG;
  if (G != 0 && G != 1 && G != 3) return QVAE_ERR_ARG;
  if (G == 3 && MS > 2) return QVAE_ERR_ARG;
  g_force[0] = MS;
  g_force[1] = NT;
  g_force[2] = SA;
  g_force[3] = SB;
  g_force[4] = mode;
  g_force[5] = G;
  return QVAE_OK;
}

int qvae_set_fused_quant(int32_t on) {
  if (on < 0 || on > 1) return QVAE_ERR_ARG;
  g_fused_quant = on != 0;
  return QVAE_OK;
}

int qvae_set_conv_cta_limit(int32_t max_ctas) {
  if (max_ctas < 0) return QVAE_ERR_ARG;
  g_cta_limit = max_ctas;
  return QVAE_OK;
}

int qvae_get_conv_tiling(const qvae_shape* shape, int32_t variant, int32_t* out8) {
  if (!out8 || variant < 0 || variant > 2) return QVAE_ERR_ARG;
  int rc = check_shape(shape);
  if (rc) return rc;
  int sms = 148, dev;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) sm_count(dev, &sms);
  cudaGetLastError();
  qvae_shape sb = *shape;
  if (variant == 2) sb.Cin *= 2;  // native precision: tiled by bytes
  Tiling t;
  if ((rc = make_tiling(sb, &t, sms, variant == 1))) return rc;
  out8[0] = t.MS;
  out8[1] = t.NT;
  out8[2] = t.SA;
  out8[3] = t.SB;
  out8[4] = t.acc_stages;
  out8[5] = t.num_tiles * t.ctas_per_tile;
  out8[6] = t.pair ? 2 : 1;
  out8[7] = t.G;
  return QVAE_OK;
}

}  // extern "C"
