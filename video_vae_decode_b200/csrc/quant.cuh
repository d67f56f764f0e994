// quant.cuh -- INT8 quantisation kernels.
//
// Scheme (ComfyUI-Qwen-VAE-Triton v0.2.0 release note, "three presets"):
// weights are symmetric INT8 with one scale per output channel, activations
// are dynamic symmetric INT8 (one scale per tensor), clip ratio 1.0 for both.
// scale = absmax / 127 and code = clamp(rint(v / scale), -127, 127) with an
// IEEE round-to-nearest divide and round-half-to-even; absmax == 0 gives
// scale 0 and all-zero codes.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace qvae {

// |bf16| ordering equals the unsigned ordering of its low 15 bits (finite
// inputs), so absmax is taken on integers and widened once at the end.
__device__ __forceinline__ uint32_t abs_bits_max2(uint32_t m, uint32_t word) {
  const uint32_t lo = word & 0x7FFFu, hi = (word >> 16) & 0x7FFFu;
  return max(m, max(lo, hi));
}

// Both 16-bit halves at once: per half, the larger of m's half and the
// magnitude (sign cleared) of the word's bf16 in that half (the same unsigned
// comparison of 15-bit magnitudes as abs_bits_max2, two values per instruction).
__device__ __forceinline__ uint32_t abs_bits_max2x(uint32_t m2, uint32_t word) {
  return __vmaxu2(m2, word & 0x7FFF7FFFu);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Rounded quotient v / s to the nearest integer (ties to even), clamped to
// [-127, 127], returned as the low byte of a float's bit pattern.
//
// The quotient is the IEEE round-to-nearest v / s.  It is computed from
// r = RN(1 / s) with one multiply and one remainder correction (Markstein's
// correctly rounded division: q0 = RN(v r), e = fma(-q0, s, v) exactly,
// q = fma(e, r, q0)); the activation tests check it code-for-code against
// the plain divide over every bf16 input for many scales.  Rounding to an
// integer adds 1.5 * 2^23: the sum lies in [2^23, 2^24) where the spacing is
// 1, so the IEEE add rounds half to even, and the low mantissa byte is the
// two's-complement code.
struct Quantizer {
  float s, r;
  bool exact;  // plain divide (tiny scales whose reciprocal overflows)
  __device__ __forceinline__ uint32_t code_byte(float v) const {
    float q;
    if (exact) {
      q = __fdiv_rn(v, s);
    } else {
      const float q0 = __fmul_rn(v, r);
      const float e = __fmaf_rn(-q0, s, v);
      q = __fmaf_rn(e, r, q0);
    }
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(q, 12582912.0f)) & 0xFFu;
  }
};

__device__ __forceinline__ Quantizer make_quantizer(float s) {
  Quantizer z;
  z.s = s;
  z.r = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
  z.exact = !(s >= 0x1p-100f);
  return z;
}

// Four bf16 (two 32-bit words) -> four packed codes.
__device__ __forceinline__ uint32_t quant4(const Quantizer& z, uint32_t w0, uint32_t w1) {
  const uint32_t c0 = z.code_byte(__uint_as_float(w0 << 16));
  const uint32_t c1 = z.code_byte(__uint_as_float(w0 & 0xFFFF0000u));
  const uint32_t c2 = z.code_byte(__uint_as_float(w1 << 16));
  const uint32_t c3 = z.code_byte(__uint_as_float(w1 & 0xFFFF0000u));
  return c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
}

template <int kThreads>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t m, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = (lane < kThreads / 32) ? red[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) red[0] = m;
  }
  __syncthreads();
  const uint32_t r = red[0];
  __syncthreads();
  return r;
}

// ------------------------------------------------------------ activations

constexpr int kActThreads = 256;
constexpr int kAbsUnroll = 8;    // 16-byte loads in flight per thread, absmax pass
constexpr int kQuantUnroll = 4;  // 32-byte (16-value) groups in flight per thread, quantise pass

// Pass 1: per-block absmax (as 15-bit magnitude codes) of a bf16 tensor.
// x is 16-byte aligned; nvec = numel / 8 full vectors; block 0 also covers the
// tail.  Each thread keeps kAbsUnroll loads in flight.  Plain cached loads:
// the most recently read part of x is still in L2 when pass 2, which walks
// the tensor backwards, starts.
__global__ void __launch_bounds__(kActThreads) act_absmax_kernel(const uint4* __restrict__ x,
                                                                  int64_t nvec,
                                                                  const uint16_t* __restrict__ xs,
                                                                  int64_t numel,
                                                                  uint32_t* __restrict__ partial,
                                                                  uint32_t* amax_word) {
  __shared__ uint32_t red[kActThreads / 32];
  grid_dependents_launch();  // the quantiser may start its prologue
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kActThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kActThreads + threadIdx.x;
  for (; i + (kAbsUnroll - 1) * stride < nvec; i += kAbsUnroll * stride) {
    uint4 v[kAbsUnroll];
#pragma unroll
    for (int u = 0; u < kAbsUnroll; ++u) v[u] = __ldg(x + i + u * stride);
#pragma unroll
    for (int u = 0; u < kAbsUnroll; ++u)
      m[u & 3] = abs_bits_max2x(abs_bits_max2x(abs_bits_max2x(abs_bits_max2x(m[u & 3], v[u].x), v[u].y), v[u].z),
                                v[u].w);
  }
  for (int j = 0; j < 4; ++j) m[j] = max(m[j] & 0xFFFFu, m[j] >> 16);  // fold the two halves
  for (; i < nvec; i += stride) {
    const uint4 a = __ldg(x + i);
    m[0] = abs_bits_max2(abs_bits_max2(abs_bits_max2(abs_bits_max2(m[0], a.x), a.y), a.z), a.w);
  }
  if (blockIdx.x == 0) {
    for (int64_t k = nvec * 8 + threadIdx.x; k < numel; k += kActThreads)
      m[0] = max(m[0], static_cast<uint32_t>(xs[k]) & 0x7FFFu);
  }
  const uint32_t mm = block_max_u32<kActThreads>(max(max(m[0], m[1]), max(m[2], m[3])), red);
  if (threadIdx.x == 0) {
    if (amax_word) {
      atomicMax(amax_word, mm);  // one maximum for the whole tensor (zeroed beforehand)
    } else {
      partial[blockIdx.x] = mm;
    }
  }
}

// Four codes from four bf16 values, two at a time on the packed fp32 pipe
// (mul / fma .rn.f32x2): the same correctly rounded quotient as code_byte
// (q0 = RN(v r), e = fma(-q0, s, v), q = fma(e, r, q0)) and the same
// round-half-even add of 1.5 * 2^23.  No clamp: |v| <= amax and
// s = RN(amax / 127) >= (amax / 127)(1 - 2^-24) give |v / s| < 127.00001, whose
// rounded quotient rounds to at most 127.  For normal, non-zero scales only
// (make_quantizer's reciprocal path).
__device__ __forceinline__ uint32_t quant4_x2(const Quantizer& z, uint32_t w0, uint32_t w1) {
  const uint64_t rr = (static_cast<uint64_t>(__float_as_uint(z.r)) << 32) | __float_as_uint(z.r);
  const uint64_t ns = (static_cast<uint64_t>(__float_as_uint(-z.s)) << 32) | __float_as_uint(-z.s);
  const uint64_t mg = 0x4B4000004B400000ull;  // 1.5 * 2^23 in both halves
  // (v0, v1) in the low / high halves: the bf16 values widened to fp32
  const uint64_t va = (static_cast<uint64_t>(w0 & 0xFFFF0000u) << 32) | (w0 << 16);
  const uint64_t vb = (static_cast<uint64_t>(w1 & 0xFFFF0000u) << 32) | (w1 << 16);
  uint64_t qa, qb, ea, eb;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(qa) : "l"(va), "l"(rr));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(qb) : "l"(vb), "l"(rr));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ea) : "l"(qa), "l"(ns), "l"(va));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(eb) : "l"(qb), "l"(ns), "l"(vb));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(qa) : "l"(ea), "l"(rr), "l"(qa));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(qb) : "l"(eb), "l"(rr), "l"(qb));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(qa) : "l"(qa), "l"(mg));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(qb) : "l"(qb), "l"(mg));
  // low bytes of the four sums, in order v0, v1 (from w0), v2, v3 (from w1)
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(qa), static_cast<uint32_t>(qa >> 32), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(qb), static_cast<uint32_t>(qb >> 32), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// 16 bf16 values (two 16-byte vectors) -> 16 codes (one 16-byte vector).
__device__ __forceinline__ uint4 quant16(const Quantizer& z, bool zero, const uint4& a, const uint4& b) {
  if (zero) return make_uint4(0u, 0u, 0u, 0u);
  return make_uint4(quant4(z, a.x, a.y), quant4(z, a.z, a.w), quant4(z, b.x, b.y), quant4(z, b.z, b.w));
}

// quant16 on the packed fp32 pipe (normal scales; tiny scales take quant16).
__device__ __forceinline__ uint4 quant16_x2(const Quantizer& z, bool zero, const uint4& a, const uint4& b) {
  if (zero) return make_uint4(0u, 0u, 0u, 0u);
  if (z.exact) return quant16(z, false, a, b);
  return make_uint4(quant4_x2(z, a.x, a.y), quant4_x2(z, a.z, a.w), quant4_x2(z, b.x, b.y), quant4_x2(z, b.z, b.w));
}

// Pass 2: reduce the partial maxima (or read the one maximum the previous
// layer's convolution accumulated), derive the scale, write INT8 codes.
// Group g (g < nvec2 = numel / 16) is 16 values: two 16-byte bf16 vectors in,
// one 16-byte code vector out.  Groups are visited from the end of the tensor
// to its start: the re-read of x begins with what pass 1 read last (still in
// L2), and the start of xq, which the convolution reads first, is written
// last.  The first loads of x are issued before waiting for pass 1 (x was
// complete before pass 1 began).  The quotients run on the packed fp32 pipe
// (quant16_x2: the same codes; the scalar form measured issue-bound, about
// 30 % slower on 100-400 MB tensors).
__global__ void __launch_bounds__(kActThreads) act_quant_kernel(
    const uint4* __restrict__ x, int64_t nvec2, const uint16_t* __restrict__ xs, int64_t numel,
    const uint32_t* __restrict__ partial, int npartial, uint4* __restrict__ xq,
    int8_t* __restrict__ xq_bytes, float* __restrict__ x_scale, uint32_t* zero_word) {
  __shared__ uint32_t red[kActThreads / 32];
  grid_dependents_launch();  // the convolution may start its prologue
  // a word the following convolution accumulates a maximum into starts at zero
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kActThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kActThreads + threadIdx.x;
  const int64_t last = nvec2 - 1;
  uint4 va[kQuantUnroll], vb[kQuantUnroll];
  const bool full = i + (kQuantUnroll - 1) * stride < nvec2;
  if (full) {
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t g = last - (i + u * stride);
      va[u] = __ldcs(x + 2 * g);
      vb[u] = __ldcs(x + 2 * g + 1);
    }
  }
  grid_dependency_wait();  // the partial maxima of the previous kernel are complete
  uint32_t m = 0;
  for (int k = threadIdx.x; k < npartial; k += kActThreads) m = max(m, partial[k]);
  m = block_max_u32<kActThreads>(m, red);
  const float amax = bf16_bits_to_f32(m) * 1.0f;  // activation clip ratio 1.0
  const float s = __fdiv_rn(amax, 127.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *x_scale = s;
  const Quantizer z = make_quantizer(s);
  const bool zero = (s == 0.0f);

  if (full) {
    while (true) {
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) xq[last - (i + u * stride)] = quant16_x2(z, zero, va[u], vb[u]);
      i += kQuantUnroll * stride;
      if (i + (kQuantUnroll - 1) * stride >= nvec2) break;
#pragma unroll
      for (int u = 0; u < kQuantUnroll; ++u) {
        const int64_t g = last - (i + u * stride);
        va[u] = __ldcs(x + 2 * g);
        vb[u] = __ldcs(x + 2 * g + 1);
      }
    }
  }
  for (; i < nvec2; i += stride) {
    const int64_t g = last - i;
    xq[g] = quant16_x2(z, zero, __ldcs(x + 2 * g), __ldcs(x + 2 * g + 1));
  }
  if (blockIdx.x == 0) {
    for (int64_t k = nvec2 * 16 + threadIdx.x; k < numel; k += kActThreads) {
      const uint32_t c = zero ? 0u : z.code_byte(bf16_bits_to_f32(xs[k]));
      xq_bytes[k] = static_cast<int8_t>(static_cast<uint8_t>(c));
    }
  }
}

// ---------------------------------------------------------------- weights

// An empty kernel launched (plainly) after the weight packer.  The
// convolution is launched as a programmatic dependent of the kernel before it
// and loads weights before it waits for that kernel; with this kernel last,
// the kernel a convolution can overlap is one that starts only after the
// packer has finished and its writes are visible.
__global__ void stream_fence_kernel() {}

constexpr int kWThreads = 256;

// One block per output channel: s_w[co] = absmax(w[co, ...]) / 127.
// w: bf16 [Cout][Cin][3][3][3] (PyTorch Conv3d layout).
__global__ void __launch_bounds__(kWThreads) weight_scale_kernel(const uint16_t* __restrict__ w,
                                                                  int Cin,
                                                                  float* __restrict__ w_scale) {
  __shared__ uint32_t red[kWThreads / 32];
  const int co = blockIdx.x;
  const int64_t per = static_cast<int64_t>(Cin) * 27;
  const uint16_t* wc = w + co * per;
  uint32_t m = 0;
  for (int64_t k = threadIdx.x; k < per; k += kWThreads) m = max(m, static_cast<uint32_t>(wc[k]) & 0x7FFFu);
  m = block_max_u32<kWThreads>(m, red);
  if (threadIdx.x == 0) w_scale[co] = __fdiv_rn(bf16_bits_to_f32(m) * 1.0f, 127.0f);  // clip 1.0
}

// Codes in the convolution's consumption order.  One thread per packed byte:
//   packed[tap][chunk][co][128]   tap = (kt * 3 + kh) * 3 + kw, chunk = 128 input channels;
// inside a 128-byte row the 16-byte group g holds channels chunk*128 + (g ^ (co & 7))*16 + [0,16)
// (the tensor cores' 128-byte swizzle, so a plain bulk copy lands in MMA layout); channels
// beyond Cin are zero.  plain (optional): [co][tap][Cin] codes for checking.
__global__ void weight_pack_kernel(const uint16_t* __restrict__ w, int Cin, int Cout, int nchunks,
                                   const float* __restrict__ w_scale, int8_t* __restrict__ packed,
                                   int8_t* __restrict__ plain) {
  const int64_t total = static_cast<int64_t>(27) * nchunks * Cout * 128;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(idx & 127);
    int64_t rest = idx >> 7;
    const int co = static_cast<int>(rest % Cout);
    rest /= Cout;
    const int chunk = static_cast<int>(rest % nchunks);
    const int tap = static_cast<int>(rest / nchunks);
    const int g = (b >> 4) ^ (co & 7);
    const int ci = chunk * 128 + g * 16 + (b & 15);
    uint32_t code = 0;
    if (ci < Cin) {
      const int kt = tap / 9, kh = (tap / 3) % 3, kw = tap % 3;
      const float v = bf16_bits_to_f32(w[((static_cast<int64_t>(co) * Cin + ci) * 3 + kt) * 9 + kh * 3 + kw]);
      const float s = w_scale[co];
      if (s != 0.0f) {
        float q = rintf(__fdiv_rn(v, s));
        q = fminf(fmaxf(q, -127.0f), 127.0f);
        code = static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu;
      }
      if (plain) plain[(static_cast<int64_t>(co) * 27 + tap) * Cin + ci] = static_cast<int8_t>(code);
    }
    packed[idx] = static_cast<int8_t>(static_cast<uint8_t>(code));
  }
}

// bf16 weights of a native-precision layer in the convolution's consumption
// order (no quantisation).  One thread per packed bf16 value:
//   packed[tap][chunk][co][64]   tap = (kt * 3 + kh) * 3 + kw, chunk = 64 input channels (128 bytes);
// inside a 128-byte row the 16-byte group g holds channels chunk*64 + (g ^ (co & 7))*8 + [0,8)
// (the same 128-byte swizzle as the INT8 packing); channels beyond Cin are zero.
__global__ void weight_pack_bf16_kernel(const uint16_t* __restrict__ w, int Cin, int Cout, int nchunks,
                                        uint16_t* __restrict__ packed) {
  const int64_t total = static_cast<int64_t>(27) * nchunks * Cout * 64;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(idx & 63);  // bf16 slot in the 128-byte row
    int64_t rest = idx >> 6;
    const int co = static_cast<int>(rest % Cout);
    rest /= Cout;
    const int chunk = static_cast<int>(rest % nchunks);
    const int tap = static_cast<int>(rest / nchunks);
    const int g = (e >> 3) ^ (co & 7);
    const int ci = chunk * 64 + g * 8 + (e & 7);
    uint16_t v = 0;
    if (ci < Cin) {
      const int kt = tap / 9, kh = (tap / 3) % 3, kw = tap % 3;
      v = w[((static_cast<int64_t>(co) * Cin + ci) * 3 + kt) * 9 + kh * 3 + kw];
    }
    packed[idx] = v;
  }
}

}  // namespace qvae
