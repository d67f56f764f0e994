// conv.cuh -- W8A8 causal 3x3x3 convolution as an implicit GEMM on the
// sm_100a tensor cores (tcgen05 kind::i8, INT32 accumulators in TMEM).
//
// What it computes (ComfyUI-Qwen-VAE-Triton v0.2.0 release note: opening
// paragraph -- an implicit-GEMM W8A8 kernel for the CausalConv3d layers; the
// "three presets" section -- INT8 x INT8 products, INT32 accumulation, FP32
// rescale, output in the activation's precision, channels_last):
//
//   acc[n,t,h,w,co] = sum_{kt,kh,kw,ci} xq[n, t+kt-2, h+kh-1, w+kw-1, ci] * wq[co, ci, kt, kh, kw]
//   out[n,t,h,w,co] = bf16_rne( float(acc) * (s_a * s_w[co]) + float(bias[co]) )
//
// with zeros outside the tensor (two leading causal frames, one pixel of
// spatial padding).  GEMM view: M = output pixels, N = Cout, K = taps x Cin.
//
// Tiling.  A CTA tile is MS sub-tiles of 128 pixels (BH rows x BW columns of
// one frame, stacked vertically) by NT output channels.  For each real
// temporal tap kt, each kw and each 128-channel chunk, one TMA box of
// (MS*BH + 2) rows x BW pixels x 128 channels is loaded once (the tensor map's
// out-of-bounds fill supplies the spatial zero padding); the three kh taps
// are then the same box read at row offsets 0, 1, 2 -- a shift of BW*128
// bytes, a whole number of 1024-byte swizzle atoms -- so the halo rows are
// shared instead of reloaded.  Temporal taps that meet a causal zero frame are
// skipped, not computed.  Weights come pre-packed in the MMA's swizzled K-major
// layout and are streamed per (tap, chunk) with plain bulk copies.
//
// Warp roles (192 threads): warp 0 issues the TMA / bulk copies, warp 1
// issues tcgen05.mma (one thread) and owns the TMEM allocation, warps 2-5 run
// the epilogue: tcgen05.ld of their 32 TMEM lanes, rescale + bias + bf16,
// 16-byte stores.  Tiles are scheduled persistently (static stride); with
// MS*NT <= 256 TMEM columns the accumulator is double-buffered so the
// epilogue of one tile overlaps the main loop of the next.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace qvae {

struct ConvArgs {
  int N, T, H, W, Cin, Cout;
  int BW, BH, MS, NT;         // tile geometry (BW * BH == 128)
  int tiles_w, tiles_h, tiles_n, num_tiles;
  int nchunks, last_ksteps;   // 128-channel chunks; 32-channel k-steps in the last one
  int SA, SB, acc_stages;     // pipeline depths
  uint32_t a_stage_bytes, b_stage_bytes, tmem_cols;
  const int8_t* wq;           // packed weights
  const float* x_scale;       // device scalar
  const float* w_scale;       // [Cout]
  const __nv_bfloat16* bias;  // [Cout] or null
  __nv_bfloat16* out;         // [N,T,H,W,Cout]
  int32_t* acc_out;           // [N,T,H,W,Cout] (accumulator mode)
  uint64_t wait_limit_ns;
};

constexpr int kConvThreads = 192;
constexpr int kMaxStages = 8;

struct TileCoord {
  int n, t, h0, w0, co0;
};

__device__ __forceinline__ TileCoord decode_tile(const ConvArgs& a, int tile) {
  TileCoord c;
  int r = tile;
  const int tn = r % a.tiles_n;
  r /= a.tiles_n;
  const int tw = r % a.tiles_w;
  r /= a.tiles_w;
  const int th = r % a.tiles_h;
  r /= a.tiles_h;
  c.t = r % a.T;
  c.n = r / a.T;
  c.h0 = th * a.MS * a.BH;
  c.w0 = tw * a.BW;
  c.co0 = tn * a.NT;
  return c;
}

template <bool kAcc32>
__global__ void __launch_bounds__(kConvThreads, 1)
    conv3d_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_x, const ConvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);

  const uint32_t a_ring = base;
  const uint32_t b_ring = a_ring + a.SA * a.a_stage_bytes;
  const uint32_t bars = b_ring + a.SB * a.b_stage_bytes;  // 8-byte mbarriers
  const uint32_t a_full = bars, a_empty = a_full + 8 * kMaxStages;
  const uint32_t b_full = a_empty + 8 * kMaxStages, b_empty = b_full + 8 * kMaxStages;
  const uint32_t acc_full = b_empty + 8 * kMaxStages, acc_empty = acc_full + 16;
  const uint32_t drain_bar = acc_empty + 16;
  uint8_t* const misc = base_ptr + (drain_bar + 8 - base);
  volatile uint32_t* const tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* const epi_smem = reinterpret_cast<float*>(misc + 16);  // 4 warps x 2 x NT floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.SA; ++i) {
      mbar_init(a_full + 8 * i, 1);
      mbar_init(a_empty + 8 * i, 1);
    }
    for (int i = 0; i < a.SB; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + 8 * i, 1);
      mbar_init(acc_empty + 8 * i, 4);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = a.wait_limit_ns;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    prefetch_tmap(&tmap_x);
    uint32_t as = 0, ap = 0, bs = 0, bp = 0;
    uint32_t a_armed = 0, a_par = 0, b_armed = 0, b_par = 0;  // per-stage bitmasks
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(a, tile);
      const int kt_lo = c.t >= 2 ? 0 : 2 - c.t;
      for (int kt = kt_lo; kt < 3; ++kt)
        for (int kw = 0; kw < 3; ++kw)
          for (int ch = 0; ch < a.nchunks; ++ch) {
            if (!mbar_wait(a_empty + 8 * as, ap ^ 1, abort_flag, limit, kErrTimeoutProducer)) goto producer_done;
            mbar_arrive_expect_tx(a_full + 8 * as, a.a_stage_bytes);
            tma_load_5d(a_ring + as * a.a_stage_bytes, &tmap_x, a_full + 8 * as, ch * 128,
                        c.w0 + kw - 1, c.h0 - 1, c.t + kt - 2, c.n);
            a_armed |= 1u << as;
            a_par = (a_par & ~(1u << as)) | (ap << as);
            if (++as == static_cast<uint32_t>(a.SA)) { as = 0; ap ^= 1; }
            for (int kh = 0; kh < 3; ++kh) {
              if (!mbar_wait(b_empty + 8 * bs, bp ^ 1, abort_flag, limit, kErrTimeoutProducer)) goto producer_done;
              const int tap = (kt * 3 + kh) * 3 + kw;
              const int8_t* src = a.wq + (static_cast<int64_t>(tap * a.nchunks + ch) * a.Cout + c.co0) * 128;
              mbar_arrive_expect_tx(b_full + 8 * bs, a.b_stage_bytes);
              bulk_load(b_ring + bs * a.b_stage_bytes, src, a.b_stage_bytes, b_full + 8 * bs);
              b_armed |= 1u << bs;
              b_par = (b_par & ~(1u << bs)) | (bp << bs);
              if (++bs == static_cast<uint32_t>(a.SB)) { bs = 0; bp ^= 1; }
            }
          }
    }
  producer_done:
    if (*abort_flag) {
      // Let every copy this thread started land before the CTA exits.
      int dummy = 0;
      for (int i = 0; i < a.SA; ++i)
        if (a_armed >> i & 1) mbar_wait(a_full + 8 * i, a_par >> i & 1, &dummy, limit, kErrTimeoutDrain);
      for (int i = 0; i < a.SB; ++i)
        if (b_armed >> i & 1) mbar_wait(b_full + 8 * i, b_par >> i & 1, &dummy, limit, kErrTimeoutDrain);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_i8(128, a.NT);
    const uint32_t row_shift = static_cast<uint32_t>(a.BW) * 128u;  // one image row of the box
    uint32_t as = 0, ap = 0, bs = 0, bp = 0, cs = 0, cp = 0;
    bool issued = false;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(a, tile);
      const int kt_lo = c.t >= 2 ? 0 : 2 - c.t;
      if (!mbar_wait(acc_empty + 8 * cs, cp ^ 1, abort_flag, limit, kErrTimeoutMma)) goto mma_done;
      tc_fence_after();
      const uint32_t d_tile = tmem_base + cs * static_cast<uint32_t>(a.MS * a.NT);
      bool first = true;
      for (int kt = kt_lo; kt < 3; ++kt)
        for (int kw = 0; kw < 3; ++kw)
          for (int ch = 0; ch < a.nchunks; ++ch) {
            if (!mbar_wait(a_full + 8 * as, ap, abort_flag, limit, kErrTimeoutMma)) goto mma_done;
            tc_fence_after();
            const int ksteps = (ch == a.nchunks - 1) ? a.last_ksteps : 4;
            const uint32_t a_stage = a_ring + as * a.a_stage_bytes;
            for (int kh = 0; kh < 3; ++kh) {
              if (!mbar_wait(b_full + 8 * bs, bp, abort_flag, limit, kErrTimeoutMma)) goto mma_done;
              tc_fence_after();
              const uint32_t b_stage = b_ring + bs * a.b_stage_bytes;
              for (int s = 0; s < a.MS; ++s) {
                const uint32_t a_rows = a_stage + static_cast<uint32_t>(s * a.BH + kh) * row_shift;
                for (int k = 0; k < ksteps; ++k) {
                  mma_i8(d_tile + static_cast<uint32_t>(s * a.NT), sw128_kmajor_desc(a_rows + 32u * k),
                         sw128_kmajor_desc(b_stage + 32u * k), idesc, (first && k == 0) ? 0u : 1u);
                  issued = true;
                }
              }
              first = false;
              mma_commit(b_empty + 8 * bs);
              if (++bs == static_cast<uint32_t>(a.SB)) { bs = 0; bp ^= 1; }
            }
            mma_commit(a_empty + 8 * as);
            if (++as == static_cast<uint32_t>(a.SA)) { as = 0; ap ^= 1; }
          }
      mma_commit(acc_full + 8 * cs);
      if (++cs == static_cast<uint32_t>(a.acc_stages)) { cs = 0; cp ^= 1; }
    }
  mma_done:
    if (*abort_flag && issued) {
      // Wait for the tensor cores to finish what was issued before TMEM is freed.
      int dummy = 0;
      mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, &dummy, limit, kErrTimeoutDrain);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;          // tile row = TMEM lane
    float* const sc = epi_smem + (warp - 2) * 2 * a.NT;
    float* const bi = sc + a.NT;
    uint32_t cs = 0, cp = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(a, tile);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full + 8 * cs, cp, abort_flag, limit, kErrTimeoutEpilogue);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      if (!kAcc32) {
        const float sa = *a.x_scale;
        for (int j = lane; j < a.NT; j += 32) {
          sc[j] = __fmul_rn(sa, a.w_scale[c.co0 + j]);
          bi[j] = a.bias ? __bfloat162float(a.bias[c.co0 + j]) : 0.0f;
        }
        __syncwarp();
      }
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + cs * static_cast<uint32_t>(a.MS * a.NT);
      for (int s = 0; s < a.MS; ++s) {
        const int h = c.h0 + s * a.BH + row / a.BW;
        const int w = c.w0 + row % a.BW;
        const bool valid = h < a.H && w < a.W;
        const int64_t pix = ((static_cast<int64_t>(c.n) * a.T + c.t) * a.H + h) * a.W + w;
        for (int cc = 0; cc < a.NT; cc += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(s * a.NT + cc), v);
          tmem_ld_wait();
          if (!valid) continue;
          if (kAcc32) {
            int4* dst = reinterpret_cast<int4*>(a.acc_out + pix * a.Cout + c.co0 + cc);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_int4(static_cast<int>(v[4 * e]), static_cast<int>(v[4 * e + 1]),
                                 static_cast<int>(v[4 * e + 2]), static_cast<int>(v[4 * e + 3]));
          } else {
            uint32_t packed[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float y0 = __fmul_rn(__int2float_rn(static_cast<int>(v[2 * e])), sc[cc + 2 * e]);
              float y1 = __fmul_rn(__int2float_rn(static_cast<int>(v[2 * e + 1])), sc[cc + 2 * e + 1]);
              y0 = __fadd_rn(y0, bi[cc + 2 * e]);
              y1 = __fadd_rn(y1, bi[cc + 2 * e + 1]);
              const __nv_bfloat162 p = __floats2bfloat162_rn(y0, y1);
              packed[e] = *reinterpret_cast<const uint32_t*>(&p);
            }
            uint4* dst = reinterpret_cast<uint4*>(a.out + pix * a.Cout + c.co0 + cc);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * cs);
      if (++cs == static_cast<uint32_t>(a.acc_stages)) { cs = 0; cp ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

// A wait that nothing satisfies: checks that a bounded wait gives up, raises
// the error word and lets the kernel return (used by the self-test entry).
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns, kErrTimeoutMma);
  __syncthreads();
}

}  // namespace qvae
