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
// Tiling.  A CTA tile is MS sub-tiles of 128 output pixels -- 16 image rows
// x 8 columns of one frame, stacked vertically -- by NT output channels.  For
// each real temporal tap kt and each 128-channel chunk, ONE TMA box of
// (16*MS + 2) rows x 10 columns x 128 channels is loaded (the tensor map's
// out-of-bounds fill supplies the zero padding).  In shared memory a pixel is
// one 128-byte line of the tensor cores' 128-byte-swizzled K-major layout, and
// an 8-pixel image row is one 8-line core-matrix group; with a group stride of
// 10 lines (the box width) every one of the nine spatial taps (kh, kw) is the
// same box read from line (kh * 10 + kw) on.  The swizzle is a function of the
// absolute shared-memory address, so any line offset is a valid operand start:
// the halo is loaded once and reused nine times.  Temporal taps that meet a
// causal zero frame are skipped, not computed.  Weights come pre-packed in the
// MMA's swizzled K-major layout and stream by 2-D TMA, G taps (1, or 3 = one
// kernel row) per pipeline stage, so the MMA warp waits and commits once per
// G taps.
//
// CTA pairs.  With kPair the kernel runs as 2-CTA clusters on the tensor
// cores' cta_group::2 path: one MMA covers M = 256 (128 pixels in each CTA)
// by NT channels; each CTA loads its own activation box and HALF of every
// weight tile (NT/2 rows), so weight traffic and shared-memory reads per
// multiply-add halve.  Every load of both CTAs is counted on the leader CTA's
// barriers; the leader issues the MMAs and its commits arrive on the barriers
// of both CTAs; each CTA's epilogue drains its own TMEM rows.  No TMA load
// uses cluster multicast.
//
// Warp roles (320 threads): warp 0 issues the TMA loads, warp 1 owns the
// TMEM allocation and runs the MMA issue loop (the whole warp; one elected
// lane issues each weight stage's tcgen05.mma sequence), warps 2-9 run the
// epilogue (two per TMEM lane quarter): tcgen05.ld of their 32 TMEM lanes,
// rescale + bias + bf16, staged through shared memory and written with TMA
// stores.  Tiles are scheduled persistently (static stride).  With MS*NT <=
// 256 TMEM columns the accumulator is double-buffered so the epilogue of one
// tile overlaps the main loop of the next; with one buffer of several
// sub-tiles, the sub-tiles are handed to the epilogue one by one (see
// mma_issue_loop).
// Launched as a programmatic dependent of the activation quantiser: the
// prologue and the first weight loads overlap its tail.
//
// Variants of the same kernel (ConvArgs): a streamed chunk whose input holds
// two carried frames in place of the causal zero frames (carry), a row band
// whose input holds halo rows in place of the top / bottom padding
// (halo_top), raw INT32 accumulators instead of the bf16 output (kAcc32), and
// the maximum |output| accumulated for the next layer's quantiser (out_amax).
//
// Native precision (conv3d_bf16_kernel).  The release note's Aggressive
// preset keeps two decoder convolutions in their original precision.  They
// run on the same body with bf16 operands: a 128-byte shared-memory line then
// holds 64 channels instead of 128 codes and one tcgen05.mma.kind::f16 step
// consumes K = 16 bf16 values (32 bytes) instead of 32 codes, so the boxes,
// rings, tap offsets and descriptors are unchanged; the accumulators are fp32
// and the epilogue computes bf16_rne(acc + bias).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include <type_traits>

#include "ptx.cuh"
#include "quant.cuh"

namespace qvae {

constexpr int kTileW = 8;       // output columns per tile = one 8-line core-matrix group
constexpr int kTileRows = 16;   // image rows per 128-pixel sub-tile
constexpr int kBoxW = kTileW + 2;
constexpr uint32_t kGroupStride = kBoxW * 128u;  // bytes between image rows of the box

struct ConvArgs {
  int N, T, H, W, Cin, Cout;
  int MS, NT;                 // sub-tiles per CTA tile, output channels per CTA tile
  int tiles_w, tiles_h, tiles_n, num_tiles;  // tiles_h counts CTA-pair row bands in pair mode
  int nchunks, last_ksteps;   // 128-byte channel chunks; 32-byte k-steps in the last one
  int chunk_elems;            // channels per 128-byte chunk: 128 (int8 codes) or 64 (bf16 values)
  int SA, SB, acc_stages;     // pipeline depths
  int G;                      // taps per weight stage (1 or 3; 9 / G stages per 128-channel chunk)
  int split;                  // per-sub-tile accumulator hand-off (one accumulator buffer, MS >= 2, SB >= 9 / G)
  int epi_bufs;               // staging buffers per epilogue warp (1 or 2)
  int carry;                  // 1: the input holds two carried frames before frame 0 (streamed chunk)
  int halo_top;               // input rows above output row 0 (a row band's halo: 0 or 1)
  uint32_t a_stage_bytes;     // activation stage stride (1024-aligned)
  uint32_t a_box_bytes;       // bytes one activation box delivers
  uint32_t b_tap_bytes;       // weight rows this CTA loads per tap x 128 B
  uint32_t b_stage_bytes;     // G x b_tap_bytes
  uint32_t tmem_cols;
  const float* x_scale;       // device scalar
  const float* w_scale;       // [Cout]
  const __nv_bfloat16* bias;  // [Cout] or null
  int32_t* acc_out;           // [N,T,H,W,Cout] (accumulator mode)
  uint32_t* out_amax;         // or null: max |bf16 output| (15-bit magnitude) accumulated here
  uint64_t wait_limit_ns;
  // quantisation in the kernel (fused variant): x is bf16, its codes are made here
  const uint32_t* x_amax;     // bf16 magnitude bits of max |x| (the scale is bf16(amax) / 127)
  float* x_scale_out;         // or null: the activation scale is written here
  int SS;                     // staging slots
  int stg_rows;               // image rows per staging slot
  int stg_groups;             // staging slots per activation box: (16 * MS + 2) / stg_rows
  uint32_t stg_slot_bytes;    // stg_rows x 10 pixels x 128 channels x 2 bytes
  uint32_t* zero_word;        // or null: a word set to zero (for a later layer's maximum)
  float one;                  // 1.0f (an operand the compiler cannot fold; see add_f32x2)
};

constexpr int kEpiWarps = 8;                        // two per TMEM lane quarter
constexpr int kConvThreads = 32 * (2 + kEpiWarps);  // producer, MMA, epilogue warps
constexpr int kCvtWarps = 2;                        // quantising warps of the fused variant
constexpr int kConvThreadsFused = kConvThreads + 32 * kCvtWarps;
constexpr int kMaxStages = 12;
constexpr int kMaxStgSlots = 8;
constexpr uint32_t kStgPixelBytes = 256;            // 128 bf16 channels of one pixel
constexpr uint32_t kEpiBufBytes = 2048;    // one epilogue staging buffer: 32 pixels x 64 B
constexpr int kAccBars = 8;                 // accumulator barriers: buffer x sub-tile

// Packed fp32 pairs (low word = first value).  RN(a * b); and RN(a + b)
// computed as fma(a, one, b) with `one` = (1.0, 1.0) from a kernel argument:
// the assembler contracts a packed multiply followed by a packed add into one
// fused multiply-add even with explicit round-to-nearest (one rounding where
// the epilogue needs two), and it cannot fold a multiplier whose value it
// does not know.
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t one, uint64_t b) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(one), "l"(b));
  return r;
}

struct TileCoord {
  int n, t, h0, w0, co0;
};

// Tile -> coordinates.  In pair mode a tile is a band of 2*MS sub-tiles
// shared by the two CTAs of a cluster; h0 is this CTA's first row.
template <bool kPair>
__device__ __forceinline__ TileCoord decode_tile(const ConvArgs& a, int tile, uint32_t rank) {
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
  const int band = a.MS * kTileRows;
  c.h0 = kPair ? (th * 2 + static_cast<int>(rank)) * band : th * band;
  c.w0 = tw * kTileW;
  c.co0 = tn * a.NT;
  return c;
}

struct MmaRings {
  uint32_t a_ring, b_ring;                       // shared-memory operand rings
  uint32_t a_full, a_empty, b_full, b_empty;     // ring barriers
  uint32_t acc_full, acc_empty;                  // accumulator barriers
  uint32_t tmem_base;
};

// One lane of a converged warp (the lowest active one).
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(p));
  return p != 0;
}

template <int N>
using IntC = std::integral_constant<int, N>;

// Calls f(IntC<k>{}) for the run-time k-step count k (1 to 4), so that the
// MMA sequence of a stage is straight-line code for every chunk width.
template <typename F>
__device__ __forceinline__ void with_ksteps(uint32_t ksteps, F&& f) {
  switch (ksteps) {
    case 4:
      f(IntC<4>{});
      break;
    case 3:
      f(IntC<3>{});
      break;
    case 2:
      f(IntC<2>{});
      break;
    default:
      f(IntC<1>{});
      break;
  }
}

// MMA issuer: the whole warp 1 of the pair's leader CTA runs the loop; lane
// 0 waits on the barriers and broadcasts the outcome, and one elected lane
// issues each stage's MMAs and its commit as straight-line code.  (Issued by
// a lone thread from run-time loops, the same MMAs measured up to twice the
// tensor pipe's cycles each at N = 96.)  Descriptors are built once; every
// operand start inside the rings is the base descriptor plus an offset in
// 16-byte units (all offsets stay inside the 14-bit start-address field).  A
// weight stage holds kG taps; per tap: kMS sub-tiles, each k-steps of 32
// bytes of K into its own accumulator.  One wait and one commit per stage.
//
// Accumulator barriers are per (buffer, sub-tile).  With a single buffer
// (split mode) the first and the last 128-channel chunk of a tile are issued
// sub-tile by sub-tile over all of the chunk's weight stages, which the ring
// holds at once: sub-tile s of the last chunk completes (and its epilogue
// starts) while the later sub-tiles still run, and sub-tile s of the next
// tile starts as soon as its epilogue has released it.  Returns false when a
// wait gave up (abort or time limit).
template <bool kBf16, bool kPair, bool kFuse, int kMS, int kG>
__device__ __forceinline__ bool mma_issue_loop(const ConvArgs& a, const MmaRings& r,
                                               volatile int* abort_flag, uint64_t limit, int first_tile,
                                               int tile_step, uint32_t rank, bool& issued) {
  const int lane = static_cast<int>(threadIdx.x & 31);
  const uint32_t idesc = kBf16 ? idesc_bf16(kPair ? 256 : 128, a.NT) : idesc_i8(kPair ? 256 : 128, a.NT);
  const uint64_t a_desc0 = sw128_kmajor_desc(r.a_ring, kGroupStride);
  const uint64_t b_desc0 = sw128_kmajor_desc(r.b_ring, 1024u);
  const uint32_t a_stage16 = a.a_stage_bytes >> 4, b_stage16 = a.b_stage_bytes >> 4;
  const uint32_t b_tap16 = a.b_tap_bytes >> 4;
  constexpr uint32_t sub16 = (kTileRows * kGroupStride) >> 4;  // one 16-row sub-tile
  constexpr int kGrp = 9 / kG;                                  // weight stages per chunk
  const uint32_t nt = static_cast<uint32_t>(a.NT);
  const uint32_t sb = static_cast<uint32_t>(a.SB);
  const bool split = a.split != 0;
  uint32_t as = 0, ap = 0, bs = 0, bp = 0, cs = 0, cp = 0;
  // phases already seen complete by a lookahead probe (a probe's result is
  // read only after the MMAs issued behind it, so its latency stays hidden)
  bool b_ready = false;    // b_full of stage bs
  bool a_ready = false;    // a_full of stage as
  bool acc_ready = false;  // the accumulator buffer of the next tile is free
  const int tiles_per_frame = a.tiles_n * a.tiles_w * a.tiles_h;
  // k-blocks (temporal tap x 128-channel chunk) of a tile: taps that meet the
  // causal zero frames are skipped
  auto tile_nkb = [&](int tile) -> int {
    const int t = a.T == 1 ? 0 : (tile / tiles_per_frame) % a.T;
    const int kt_lo = (a.carry || t >= 2) ? 0 : 2 - t;
    return (3 - kt_lo) * a.nchunks;
  };
  auto probe = [&](uint32_t bar, uint32_t parity) -> int {
    return lane == 0 ? (mbar_test_wait(bar, parity) ? 1 : 0) : 0;
  };
  auto seen = [&](int pr) -> bool { return __shfl_sync(0xFFFFFFFFu, pr, 0) != 0; };
  // lane 0 waits; the warp takes its outcome
  auto wait = [&](uint32_t bar, uint32_t parity, bool cluster_scope) -> bool {
    int ok = 1;
    if (lane == 0) {
      ok = cluster_scope ? mbar_wait_cluster(bar, parity, abort_flag, limit, kErrTimeoutMma)
                         : mbar_wait(bar, parity, abort_flag, limit, kErrTimeoutMma);
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    __syncwarp();
    return ok != 0;
  };
  // issued by the elected lane only
  auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t acc) {
    if (kBf16) {
      if (kPair) {
        mma_bf16_pair(d, ad, bd, idesc, acc);
      } else {
        mma_bf16(d, ad, bd, idesc, acc);
      }
    } else if (kPair) {
      mma_i8_pair(d, ad, bd, idesc, acc);
    } else {
      mma_i8(d, ad, bd, idesc, acc);
    }
  };
  auto commit_raw = [&](uint32_t bar) {
    if (kPair) {
      mma_commit_pair_multicast(bar, 0x3);
    } else {
      mma_commit(bar);
    }
  };
  // a commit issued by one elected lane of the warp
  auto commit = [&](uint32_t bar) {
    if (elect_one()) commit_raw(bar);
    __syncwarp();
  };
  (void)rank;
  for (int tile = first_tile; tile < a.num_tiles; tile += tile_step) {
    const int nkb = tile_nkb(tile);
    const uint32_t d_tile = r.tmem_base + cs * static_cast<uint32_t>(kMS) * nt;
    const uint32_t accb = cs * static_cast<uint32_t>(kMS);  // this buffer's first barrier index
    if (!check_bounds((cs + 1u) * static_cast<uint32_t>(kMS) * nt <= a.tmem_cols &&
                      accb + static_cast<uint32_t>(kMS) <= static_cast<uint32_t>(kAccBars))) {
      *abort_flag = 1;
      return false;
    }
    if (!split) {
      // the epilogue warps release a buffer's sub-tiles in order: the last one's
      // barrier completing implies the others'
      if (!acc_ready && !wait(r.acc_empty + 8 * (accb + kMS - 1), cp ^ 1, false)) return false;
      tc_fence_after();
    }
    acc_ready = false;
    uint32_t acc = 0;  // the tile's first MMA overwrites the accumulator
    for (int kb = 0; kb < nkb; ++kb) {
      const int ch = kb % a.nchunks;
      // the fused variant's A stages are written by threads of both CTAs of a pair
      if (!a_ready && !wait(r.a_full + 8 * as, ap, kFuse && kPair)) return false;
      tc_fence_after();
      a_ready = false;
      const uint32_t ksteps = (ch == a.nchunks - 1) ? static_cast<uint32_t>(a.last_ksteps) : 4u;
      const uint64_t a_stage = a_desc0 + as * a_stage16;
      const bool first = kb == 0, last = kb == nkb - 1;
      if (split && (first || last)) {
        // sub-tile by sub-tile over the chunk's kGrp stages (all resident)
        uint32_t st = bs, sp = bp;
#pragma unroll
        for (int s = 0; s < kMS; ++s) {
          if (first) {
            if (!wait(r.acc_empty + 8 * s, cp ^ 1, false)) return false;
            tc_fence_after();
          }
          uint32_t acc_s = first ? 0u : 1u;
          st = bs;
          sp = bp;
          for (int grp = 0; grp < kGrp; ++grp) {
            if (s == 0) {
              if (!wait(r.b_full + 8 * st, sp, false)) return false;
              tc_fence_after();
            }
            const uint64_t b_stage = b_desc0 + st * b_stage16;
            const uint32_t acc0 = acc_s;
            if (elect_one()) {
              with_ksteps(ksteps, [&](auto KS) {
                constexpr int ks = decltype(KS)::value;
                uint32_t acc_l = acc0;
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                  const uint32_t tap9 = static_cast<uint32_t>(grp * kG + g);
                  const uint32_t kh = tap9 / 3u, kw = tap9 % 3u;
                  const uint64_t a_tap = a_stage + ((kh * kGroupStride + kw * 128u) >> 4) + s * sub16;
                  const uint64_t b_tap = b_stage + g * b_tap16;
#pragma unroll
                  for (int k = 0; k < ks; ++k)  // 32 bytes of K = 2 units
                    mma(d_tile + s * nt, a_tap + 2 * k, b_tap + 2 * k, k == 0 ? acc_l : 1u);
                  acc_l = 1u;
                }
              });
              if (s == kMS - 1) commit_raw(r.b_empty + 8 * st);
            }
            __syncwarp();
            acc_s = 1u;
            issued = true;
            if (++st == sb) { st = 0; sp ^= 1; }
          }
          if (last) commit(r.acc_full + 8 * s);
        }
        bs = st;
        bp = sp;
        b_ready = false;
        acc = 1u;
      } else {
        for (int grp = 0; grp < kGrp; ++grp) {
          if (!b_ready && !wait(r.b_full + 8 * bs, bp, false)) return false;
          tc_fence_after();
          // lookahead: the next weight stage; on the chunk's last stage the next
          // activation stage and, on the tile's last, the next accumulator buffer
          const uint32_t nbs = (bs + 1 == sb) ? 0u : bs + 1;
          const uint32_t nbp = (bs + 1 == sb) ? bp ^ 1u : bp;
          const int pr_b = probe(r.b_full + 8 * nbs, nbp);
          int pr_a = 0, pr_acc = 0;
          if (grp == kGrp - 1) {
            const uint32_t nas = (as + 1 == static_cast<uint32_t>(a.SA)) ? 0u : as + 1;
            const uint32_t nap = (as + 1 == static_cast<uint32_t>(a.SA)) ? ap ^ 1u : ap;
            if (!kFuse || !kPair) pr_a = probe(r.a_full + 8 * nas, nap);
            if (last && !split) {
              const uint32_t ncs = (cs + 1 == static_cast<uint32_t>(a.acc_stages)) ? 0u : cs + 1;
              const uint32_t ncp = (cs + 1 == static_cast<uint32_t>(a.acc_stages)) ? cp ^ 1u : cp;
              pr_acc = probe(r.acc_empty + 8 * (ncs * kMS + kMS - 1), ncp ^ 1u);
            }
          }
          const uint64_t b_stage = b_desc0 + bs * b_stage16;
          // one elected lane issues the stage's MMAs as straight-line code
          // (an election per MMA measured 18-27 % slower on the Cout = 96 layers)
          const uint32_t acc0 = acc;
          if (elect_one()) {
            with_ksteps(ksteps, [&](auto KS) {
              constexpr int ks = decltype(KS)::value;
              uint32_t acc_l = acc0;
#pragma unroll
              for (int g = 0; g < kG; ++g) {
                const uint32_t tap9 = static_cast<uint32_t>(grp * kG + g);
                const uint32_t kh = tap9 / 3u, kw = tap9 % 3u;
                // tap (kh, kw) of sub-tile s starts at box line (s*16 + kh)*10 + kw
                const uint64_t a_tap = a_stage + ((kh * kGroupStride + kw * 128u) >> 4);
                const uint64_t b_tap = b_stage + g * b_tap16;
#pragma unroll
                for (int s = 0; s < kMS; ++s) {
#pragma unroll
                  for (int k = 0; k < ks; ++k)  // 32 bytes of K = 2 units
                    mma(d_tile + s * nt, a_tap + s * sub16 + 2 * k, b_tap + 2 * k, k == 0 ? acc_l : 1u);
                }
                acc_l = 1u;
              }
            });
            commit_raw(r.b_empty + 8 * bs);
          }
          __syncwarp();
          acc = 1u;
          issued = true;
          if (++bs == sb) { bs = 0; bp ^= 1; }
          b_ready = seen(pr_b);
          if (grp == kGrp - 1) {
            a_ready = seen(pr_a);
            acc_ready = seen(pr_acc);
          }
        }
      }
      commit(r.a_empty + 8 * as);
      if (++as == static_cast<uint32_t>(a.SA)) { as = 0; ap ^= 1; }
    }
    if (!split) {
#pragma unroll
      for (int s = 0; s < kMS; ++s) commit(r.acc_full + 8 * (accb + s));
    }
    if (++cs == static_cast<uint32_t>(a.acc_stages)) { cs = 0; cp ^= 1; }
  }
  return true;
}

// The body of both convolution kernels.  kBf16: the operands are bf16 values
// (kind::f16, fp32 accumulators, output bf16(acc + bias)); otherwise INT8
// codes (kind::i8, INT32 accumulators, output bf16(acc * scale + bias)).  In
// shared memory both are 128-byte lines per pixel -- 128 codes or 64 bf16
// channels -- and one MMA step consumes 32 bytes of K, so the tiling, the
// rings and the tap offsets are the same.
//
// kFuse (INT8 only): x arrives as bf16 and is quantised inside the kernel.
// Two more warps stream row groups of the bf16 input box into a small staging
// ring by TMA and write the codes of each 16-channel group, in the MMA's
// swizzled layout, into the activation ring -- the same codes as the
// activation quantiser, with the scale bf16(amax) / 127 taken from one device
// word.  The producer then loads weights only.
template <bool kBf16, bool kAcc32, bool kPair, bool kFuse>
__device__ __forceinline__ void conv3d_body(const CUtensorMap& tmap_x, const CUtensorMap& tmap_w,
                                            const CUtensorMap& tmap_out, const ConvArgs& a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);

  const uint32_t a_ring = base;
  const uint32_t b_ring = a_ring + a.SA * a.a_stage_bytes;
  const uint32_t stg_ring = b_ring + a.SB * a.b_stage_bytes;                     // fused: bf16 row groups
  const uint32_t epi_stage = stg_ring + (kFuse ? a.SS * a.stg_slot_bytes : 0u);  // 1024-aligned
  const uint32_t bars = epi_stage + kEpiWarps * a.epi_bufs * kEpiBufBytes;  // 8-byte mbarriers
  const uint32_t a_full = bars, a_empty = a_full + 8 * kMaxStages;
  const uint32_t b_full = a_empty + 8 * kMaxStages, b_empty = b_full + 8 * kMaxStages;
  const uint32_t acc_full = b_empty + 8 * kMaxStages, acc_empty = acc_full + 8 * kAccBars;
  // stg_done: per staging slot, a running count of quantising-warp passes over it (a plain word, 8 bytes apart)
  const uint32_t stg_full = acc_empty + 8 * kAccBars, stg_done = stg_full + 8 * kMaxStgSlots;
  const uint32_t drain_bar = stg_done + 8 * kMaxStgSlots;
  uint8_t* const misc = base_ptr + (drain_bar + 8 - base);
  volatile uint32_t* const tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  // NT scales then NT biases, shared by the epilogue warps, 16-byte aligned for vector loads
  float* const epi_smem = reinterpret_cast<float*>(base_ptr + ((drain_bar + 8 + 16 + 15 - base) & ~15u));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;      // 0 = leader of the pair
  const bool leader = rank == 0;
  const int first_tile = kPair ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int tile_step = kPair ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);

  // Start the tensor-map descriptor fetches before anything else.
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
  }
  if (threadIdx.x == 64 && !kAcc32) prefetch_tmap(&tmap_out);
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.SA; ++i) {
      // fused: one arrive per quantising warp (of both CTAs of a pair)
      mbar_init(a_full + 8 * i, kFuse ? kCvtWarps * (kPair ? 2 : 1) : 1);
      mbar_init(a_empty + 8 * i, 1);
    }
    if (kFuse) {
      for (int i = 0; i < a.SS; ++i) {
        mbar_init(stg_full + 8 * i, 1);
        asm volatile("st.shared.u32 [%0], 0;" ::"r"(stg_done + 8 * i) : "memory");
      }
    }
    for (int i = 0; i < a.SB; ++i) {
      mbar_init(b_full + 8 * i, 1);
      mbar_init(b_empty + 8 * i, 1);
    }
    for (int i = 0; i < kAccBars; ++i) {
      mbar_init(acc_full + 8 * i, 1);
      mbar_init(acc_empty + 8 * i, kPair ? 2 * kEpiWarps : kEpiWarps);  // one arrive per epilogue warp (of both CTAs)
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), a.tmem_cols);
    } else {
      tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), a.tmem_cols);
    }
  }
  tc_fence_before();
  if (kPair) {
    cluster_sync();  // both CTAs' barriers exist before either signals the other
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = a.wait_limit_ns;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // Weights do not depend on the preceding kernel: the first weight stages
    // are filled before waiting for the activation codes.
    uint32_t as = 0, ap = 0, bs = 0, bp = 0;
    uint32_t a_armed = 0, a_par = 0, b_armed = 0, b_par = 0;  // per-stage bitmasks
    const uint32_t tx_mult = kPair ? 2u : 1u;                 // bytes both CTAs deliver
    int preissued = 0;
    const int ngrp = 9 / a.G;  // weight stages per 128-channel chunk
    auto load_b = [&](const TileCoord& c, int kt, int ch, int grp) -> bool {
      if (!mbar_wait(b_empty + 8 * bs, bp ^ 1, abort_flag, limit, kErrTimeoutProducer)) return false;
      const uint32_t bar = b_full + 8 * bs;
      if (leader) mbar_arrive_expect_tx(bar, a.b_stage_bytes * tx_mult);
      for (int g = 0; g < a.G; ++g) {
        const int tap = kt * 9 + grp * a.G + g;  // (kt * 3 + kh) * 3 + kw
        const int row = (tap * a.nchunks + ch) * a.Cout + c.co0 + static_cast<int>(rank) * (a.NT / 2);
        const uint32_t dst = b_ring + bs * a.b_stage_bytes + static_cast<uint32_t>(g) * a.b_tap_bytes;
        const int rows = kPair ? a.NT / 2 : a.NT;
        if (!check_bounds(tap >= 0 && tap < 27 && ch >= 0 && ch < a.nchunks && row >= 0 &&
                          row + rows <= 27 * a.nchunks * a.Cout &&
                          dst + a.b_tap_bytes <= b_ring + static_cast<uint32_t>(a.SB) * a.b_stage_bytes))
          continue;
        if (kPair) {
          tma_load_2d_pair(dst, &tmap_w, map_to_cta(bar, 0), 0, row);
        } else {
          tma_load_2d(dst, &tmap_w, bar, 0, row);
        }
      }
      b_armed |= 1u << bs;
      b_par = (b_par & ~(1u << bs)) | (bp << bs);
      if (++bs == static_cast<uint32_t>(a.SB)) { bs = 0; bp ^= 1; }
      return true;
    };
    bool waited = false;
    for (int tile = first_tile; tile < a.num_tiles; tile += tile_step) {
      const TileCoord c = decode_tile<kPair>(a, tile, rank);
      const int kt_lo = (a.carry || c.t >= 2) ? 0 : 2 - c.t;
      const int nkb = (3 - kt_lo) * a.nchunks;
      for (int kb = 0; kb < nkb; ++kb) {
        const int kt = kt_lo + kb / a.nchunks, ch = kb % a.nchunks;
        const int frame = c.t + kt - 2 + 2 * a.carry;  // input frame of temporal tap kt
        if (!waited) {
          for (; preissued < a.SB && preissued < ngrp; ++preissued)
            if (!load_b(c, kt, ch, preissued)) goto producer_done;
          if (!kFuse) grid_dependency_wait();
          waited = true;
        }
        if (!kFuse) {
          if (!mbar_wait(a_empty + 8 * as, ap ^ 1, abort_flag, limit, kErrTimeoutProducer)) goto producer_done;
          const uint32_t bar = a_full + 8 * as;
          if (leader) mbar_arrive_expect_tx(bar, a.a_box_bytes * tx_mult);
          // the channel coordinate (the box's innermost) must sit on a 16-byte boundary
          if (!check_bounds(ch >= 0 && ch < a.nchunks && (ch * 128) % 16 == 0 && frame >= 0 &&
                            frame < a.T + 2 * a.carry && c.n >= 0 && c.n < a.N && c.w0 >= 0 && c.w0 < a.W &&
                            c.h0 >= 0 && a.a_box_bytes <= a.a_stage_bytes && as < static_cast<uint32_t>(a.SA))) {
          } else if (kPair) {
            tma_load_5d_pair(a_ring + as * a.a_stage_bytes, &tmap_x, map_to_cta(bar, 0), ch * a.chunk_elems,
                             c.w0 - 1, c.h0 - 1 + a.halo_top, frame, c.n);
          } else {
            tma_load_5d(a_ring + as * a.a_stage_bytes, &tmap_x, bar, ch * a.chunk_elems, c.w0 - 1,
                        c.h0 - 1 + a.halo_top, frame, c.n);
          }
          a_armed |= 1u << as;
          a_par = (a_par & ~(1u << as)) | (ap << as);
          if (++as == static_cast<uint32_t>(a.SA)) { as = 0; ap ^= 1; }
        }
        (void)frame;
        for (int i = preissued; i < ngrp; ++i)
          if (!load_b(c, kt, ch, i)) goto producer_done;
        preissued = 0;
      }
    }
  producer_done:
    if (*abort_flag && leader) {
      // Let every copy counted on this CTA's barriers land before it exits.
      int dummy = 0;
      for (int i = 0; i < a.SA; ++i)
        if (a_armed >> i & 1) mbar_wait(a_full + 8 * i, a_par >> i & 1, &dummy, limit, kErrTimeoutDrain);
      for (int i = 0; i < a.SB; ++i)
        if (b_armed >> i & 1) mbar_wait(b_full + 8 * i, b_par >> i & 1, &dummy, limit, kErrTimeoutDrain);
    }
  } else if (warp == 1 && leader) {
    // ---------------------------------------------------------- MMA issuer
    // One instantiation per (sub-tile count, taps per stage), so that the
    // MMA sequence of a stage is straight-line code.
    MmaRings r{a_ring, b_ring, a_full, a_empty, b_full, b_empty, acc_full, acc_empty, tmem_base};
    bool issued = false;
    bool ok;
    auto run = [&](auto ms, auto g) {
      return mma_issue_loop<kBf16, kPair, kFuse, decltype(ms)::value, decltype(g)::value>(
          a, r, abort_flag, limit, first_tile, tile_step, rank, issued);
    };
    using G1 = std::integral_constant<int, 1>;
    using G3 = std::integral_constant<int, 3>;
    switch (a.MS * 4 + a.G) {
      case 1 * 4 + 3:
        ok = run(std::integral_constant<int, 1>{}, G3{});
        break;
      case 2 * 4 + 3:
        ok = run(std::integral_constant<int, 2>{}, G3{});
        break;
      case 1 * 4 + 1:
        ok = run(std::integral_constant<int, 1>{}, G1{});
        break;
      case 2 * 4 + 1:
        ok = run(std::integral_constant<int, 2>{}, G1{});
        break;
      case 3 * 4 + 1:
        ok = run(std::integral_constant<int, 3>{}, G1{});
        break;
      default:
        ok = run(std::integral_constant<int, 4>{}, G1{});
        break;
    }
    if (!ok && issued && lane == 0 && *abort_flag) {
      // Wait for the tensor cores to finish what was issued before TMEM is freed.
      int dummy = 0;
      if (kPair) {
        mma_commit_pair(drain_bar);
      } else {
        mma_commit(drain_bar);
      }
      mbar_wait(drain_bar, 0, &dummy, limit, kErrTimeoutDrain);
    }
    __syncwarp();
  } else if (kFuse && warp >= 2 + kEpiWarps) {
    // ----------------------------------------------------------- quantisers
    // The activation boxes of the fused variant, in the MMA's order: each
    // box (tile, temporal tap, 128-channel chunk) is 16*MS + 2 rows x 10
    // columns of bf16 pixels, brought in as row groups of stg_rows rows by
    // TMA into the staging ring (SS groups in flight) and turned into codes in
    // the 128-byte-swizzled K-major layout of the activation ring.  Rows and
    // columns beyond the image arrive as zeros from the tensor map and give
    // code 0.  Each lane converts one 16-byte piece (8 channels) of a pixel
    // (consecutive lanes read consecutive pieces: no bank conflicts); lanes
    // 2k and 2k + 1 hold one 16-channel group and the even one stores it.
    // The warp that finishes a staging slot last refills it with the group SS
    // positions ahead.  When a box is complete each warp fences its shared-
    // memory writes for the tensor cores and arrives on the (leader's) a_full.
    const int cw = warp - (2 + kEpiWarps);
    const int ct = cw * 32 + lane;
    struct Pos {
      int tile, kb, g, nkb, kt_lo;
      TileCoord c;
    };
    auto start = [&](Pos& p, int tile) {
      p.tile = tile;
      p.kb = 0;
      p.g = 0;
      if (tile < a.num_tiles) {
        p.c = decode_tile<kPair>(a, tile, rank);
        p.kt_lo = (a.carry || p.c.t >= 2) ? 0 : 2 - p.c.t;
        p.nkb = (3 - p.kt_lo) * a.nchunks;
      }
    };
    auto advance = [&](Pos& p) {
      if (++p.g < a.stg_groups) return;
      p.g = 0;
      if (++p.kb < p.nkb) return;
      start(p, p.tile + tile_step);
    };
    // the TMA load of position p into staging slot `slot`
    auto issue = [&](const Pos& p, uint32_t slot) {
      const int kt = p.kt_lo + p.kb / a.nchunks, ch = p.kb % a.nchunks;
      const int frame = p.c.t + kt - 2 + 2 * a.carry;
      const uint32_t bar = stg_full + 8 * slot;
      mbar_arrive_expect_tx(bar, a.stg_slot_bytes);
      if (!check_bounds(ch >= 0 && ch < a.nchunks && frame >= 0 && frame < a.T + 2 * a.carry && p.c.n >= 0 &&
                        p.c.n < a.N && p.c.w0 >= 0 && p.c.w0 < a.W && slot < static_cast<uint32_t>(a.SS) &&
                        (p.g + 1) * a.stg_rows <= 16 * a.MS + 2))
        return;
      tma_load_5d(stg_ring + slot * a.stg_slot_bytes, &tmap_x, bar, ch * 128, p.c.w0 - 1,
                  p.c.h0 - 1 + a.halo_top + p.g * a.stg_rows, frame, p.c.n);
    };
    grid_dependency_wait();  // x and its maximum are final
    const float sa = __fdiv_rn(bf16_bits_to_f32(__ldcg(a.x_amax) & 0x7FFFu) * 1.0f, 127.0f);  // clip ratio 1.0
    const Quantizer z = make_quantizer(sa);
    const bool zero_scale = sa == 0.0f;
    if (ct == 0 && blockIdx.x == 0) {
      if (a.x_scale_out) *a.x_scale_out = sa;
      if (a.zero_word) *a.zero_word = 0u;
    }
    Pos cur, pf;
    start(cur, first_tile);
    start(pf, first_tile);
    uint32_t stg_armed = 0, stg_par = 0;  // (lane 0 of the issuing warp) slots with a load in flight
    for (uint32_t k = 0; k < static_cast<uint32_t>(a.SS) && pf.tile < a.num_tiles; ++k) {
      if (ct == 0) {
        issue(pf, k);
        stg_armed |= 1u << k;
      }
      advance(pf);
    }
    uint32_t slot = 0, sp = 0, as = 0, ap = 0;
    const int lines = a.stg_rows * kBoxW;
    bool ok = true;
    // 8 bf16 values -> 8 codes (two words)
    auto codes8 = [&](const uint4& v) -> uint2 {
      if (zero_scale) return make_uint2(0u, 0u);
      if (z.exact) return make_uint2(quant4(z, v.x, v.y), quant4(z, v.z, v.w));
      return make_uint2(quant4_x2(z, v.x, v.y), quant4_x2(z, v.z, v.w));
    };
    while (cur.tile < a.num_tiles) {
      const int ch = cur.kb % a.nchunks;
      const int np = (ch == a.nchunks - 1) ? 4 * a.last_ksteps : 16;  // 8-channel pieces the MMA reads
      const uint32_t a_st = a_ring + as * a.a_stage_bytes;
      int waited = 1;
      if (lane == 0) {
        if (cur.g == 0) waited = mbar_wait(a_empty + 8 * as, ap ^ 1, abort_flag, limit, kErrTimeoutConvert);
        if (waited) waited = mbar_wait(stg_full + 8 * slot, sp, abort_flag, limit, kErrTimeoutConvert);
      }
      if (!__shfl_sync(0xFFFFFFFFu, waited, 0)) {
        ok = false;
        break;
      }
      __syncwarp();  // lane 0's acquire covers the whole warp's accesses
      const uint32_t src = stg_ring + slot * a.stg_slot_bytes;
      const int line0 = cur.g * lines;
      const int total = lines * np;
      for (int base = 0; base < total; base += 32 * kCvtWarps) {
        const int idx = base + ct;
        const bool valid = idx < total;
        const int i = idx / np, p = idx - i * np;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (valid)
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(src + static_cast<uint32_t>(i) * kStgPixelBytes + static_cast<uint32_t>(p) * 16u));
        const uint2 c = codes8(v);
        const uint32_t ox = __shfl_xor_sync(0xFFFFFFFFu, c.x, 1), oy = __shfl_xor_sync(0xFFFFFFFFu, c.y, 1);
        if (valid && (p & 1) == 0) {
          const uint32_t L = static_cast<uint32_t>(line0 + i), u = static_cast<uint32_t>(p >> 1);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_st + L * 128u + ((u ^ (L & 7u)) << 4)),
                       "r"(c.x), "r"(c.y), "r"(ox), "r"(oy)
                       : "memory");
        }
      }
      __syncwarp();
      if (lane == 0) {
        // the last warp done with this slot's current load refills it (the other warps' reads are ordered before)
        uint32_t prev;
        asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "r"(stg_done + 8 * slot)
                     : "memory");
        if (prev % kCvtWarps == kCvtWarps - 1) {
          fence_proxy_async_smem();
          if (pf.tile < a.num_tiles) {
            issue(pf, slot);
            stg_armed |= 1u << slot;
            stg_par = (stg_par & ~(1u << slot)) | ((sp ^ 1u) << slot);
          } else {
            stg_armed &= ~(1u << slot);
          }
        } else {
          stg_armed &= ~(1u << slot);  // the other warp owns the refill
        }
      }
      advance(pf);
      if (++slot == static_cast<uint32_t>(a.SS)) { slot = 0; sp ^= 1; }
      if (cur.g == a.stg_groups - 1) {
        // the box is complete: make the codes visible to the tensor cores
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (kPair) {
            mbar_arrive_cluster(map_to_cta(a_full + 8 * as, 0));
          } else {
            mbar_arrive(a_full + 8 * as);
          }
        }
        if (++as == static_cast<uint32_t>(a.SA)) { as = 0; ap ^= 1; }
      }
      advance(cur);
    }
    if (lane == 0 && *abort_flag) {
      // let the staging loads this warp issued and that are still in flight land before the CTA exits
      int dummy = 0;
      for (int i = 0; i < a.SS; ++i)
        if (stg_armed >> i & 1) mbar_wait(stg_full + 8 * i, stg_par >> i & 1, &dummy, limit, kErrTimeoutDrain);
    }
    (void)ok;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // A warp may read only the TMEM lane quarter warp % 4; lane quarter q holds
    // tile rows 4q..4q+3 x 8 columns.  Two warps share each quarter: a
    // sub-tile's 32-channel slices alternate between them.  Sub-tiles are
    // taken in order, each as soon as its accumulator is complete, and handed
    // back to the MMA issuer when read.  Each slice is converted, staged in
    // shared memory (64-byte swizzle; one or two buffers per warp) and written
    // by one TMA store of a 32 x 8 x 4 box, which also drops the rows and
    // columns beyond the image edge.  The TMEM load of a warp's next slice is in flight while the
    // current one is converted.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int nsl = a.NT >> 5;
    float* const sc = epi_smem;
    float* const bi = sc + a.NT;
    const uint32_t stage = epi_stage + static_cast<uint32_t>((warp - 2) * a.epi_bufs) * kEpiBufBytes;
    uint32_t buf = 0;
    const uint32_t empty_leader = kPair ? map_to_cta(acc_empty, 0) : acc_empty;
    uint32_t cs = 0, cp = 0;
    int scale_co0 = -1;
    uint32_t out_max = 0;  // largest |output| written by this lane (bf16 magnitude bits)
    bool dead = false;  // a wait gave up: keep pace with the other warps' table barriers, do no work
    // Scale and bias table for output channels co0..co0+NT-1.  Every epilogue
    // warp sees the same tiles, so all of them take part; the first barrier
    // lets the previous tile's slices finish reading the old table.
    auto fill_table = [&](int co0) {
      named_barrier_sync(1, 32 * kEpiWarps);
      const float sa = kBf16   ? 1.0f
                       : kFuse ? __fdiv_rn(bf16_bits_to_f32(__ldcg(a.x_amax) & 0x7FFFu) * 1.0f, 127.0f)
                               : *a.x_scale;
      for (int j = (warp - 2) * 32 + lane; j < a.NT; j += 32 * kEpiWarps) {
        sc[j] = kBf16 ? 1.0f : __fmul_rn(sa, a.w_scale[co0 + j]);
        bi[j] = a.bias ? __bfloat162float(a.bias[co0 + j]) : 0.0f;
      }
      scale_co0 = co0;
      named_barrier_sync(1, 32 * kEpiWarps);
    };
    grid_dependency_wait();  // the activation scale is final
    for (int tile = first_tile; tile < a.num_tiles; tile += tile_step) {
      const TileCoord c = decode_tile<kPair>(a, tile, rank);
      if (!kAcc32 && c.co0 != scale_co0) fill_table(c.co0);  // before the accumulators are ready
      const uint32_t accb = cs * static_cast<uint32_t>(a.MS);
      const uint32_t t_buf = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + accb * static_cast<uint32_t>(a.NT);
      for (int s = 0; s < a.MS && !dead; ++s) {
        int ok = 1;
        // in the fused variant the quantising warps share these warps' SM
        // sub-partitions: poll with a back-off instead of spinning
        if (lane == 0)
          ok = mbar_wait(acc_full + 8 * (accb + s), cp, abort_flag, limit, kErrTimeoutEpilogue, kFuse ? 200u : 0u);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) {
          dead = true;
          break;
        }
        tc_fence_after();
        const uint32_t t_sub = t_buf + static_cast<uint32_t>(s * a.NT);
        if (!check_bounds((accb + static_cast<uint32_t>(s) + 1u) * static_cast<uint32_t>(a.NT) <= a.tmem_cols)) {
          dead = true;
          break;
        }
        auto issue = [&](int jj, uint32_t(&v)[32]) { tmem_ld_32x32b_x32(t_sub + static_cast<uint32_t>(jj << 5), v); };
        auto process = [&](int jj, const uint32_t(&v)[32]) {
          const int cc = jj << 5;
          if (kAcc32) {
            const int h = c.h0 + s * kTileRows + row / kTileW;
            const int w = c.w0 + row % kTileW;
            if (h < a.H && w < a.W && check_bounds(c.co0 + cc + 32 <= a.Cout && c.n < a.N && c.t < a.T)) {
              const int64_t pix = ((static_cast<int64_t>(c.n) * a.T + c.t) * a.H + h) * a.W + w;
              int4* dst = reinterpret_cast<int4*>(a.acc_out + pix * a.Cout + c.co0 + cc);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_int4(static_cast<int>(v[4 * e]), static_cast<int>(v[4 * e + 1]),
                                   static_cast<int>(v[4 * e + 2]), static_cast<int>(v[4 * e + 3]));
            }
          } else {
            // scale and bias pairs (channels 2i, 2i + 1) as packed fp32
            const uint64_t one2 = (static_cast<uint64_t>(__float_as_uint(a.one)) << 32) | __float_as_uint(a.one);
            const uint64_t* sc2 = reinterpret_cast<const uint64_t*>(sc + cc);
            const uint64_t* bi2 = reinterpret_cast<const uint64_t*>(bi + cc);
            uint32_t packed[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              // two channels at a time on the packed fp32 pipe:
              // y = float(acc) * scale, rounded, then + bias, rounded (the
              // explicit .rn forms are never contracted into an FMA)
              uint64_t y;
              if (kBf16) {  // fp32 accumulators: y = acc + bias
                y = add_f32x2((static_cast<uint64_t>(v[2 * e + 1]) << 32) | v[2 * e], one2, bi2[e]);
              } else {
                const uint64_t f = (static_cast<uint64_t>(__float_as_uint(__int2float_rn(static_cast<int>(v[2 * e + 1])))) << 32) |
                                   __float_as_uint(__int2float_rn(static_cast<int>(v[2 * e])));
                y = add_f32x2(mul_f32x2(f, sc2[e]), one2, bi2[e]);
              }
              const __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(static_cast<uint32_t>(y)),
                                                              __uint_as_float(static_cast<uint32_t>(y >> 32)));
              packed[e] = *reinterpret_cast<const uint32_t*>(&p2);
            }
            if (a.out_amax) {
              // the next layer's activation absmax, taken on what is written
              const int h = c.h0 + s * kTileRows + row / kTileW;
              const int w = c.w0 + row % kTileW;
              if (h < a.H && w < a.W) {
#pragma unroll
                for (int e = 0; e < 16; ++e) out_max = max(out_max, max(packed[e] & 0x7FFFu, (packed[e] >> 16) & 0x7FFFu));
              }
            }
            // the store issued epi_bufs slices ago read this buffer: let it finish
            if (lane == 0) {
              if (a.epi_bufs == 2) {
                bulk_wait_group_read<1>();
              } else {
                bulk_wait_group_read<0>();
              }
            }
            __syncwarp();
            const uint32_t sbuf = stage + buf * kEpiBufBytes;
            const uint32_t line = sbuf + static_cast<uint32_t>(lane) * 64u;
            const uint32_t swz = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(line + ((k ^ swz) << 4)),
                           "r"(packed[4 * k]), "r"(packed[4 * k + 1]), "r"(packed[4 * k + 2]),
                           "r"(packed[4 * k + 3])
                           : "memory");
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              // a box that starts below the last row is clipped whole by the tensor map
              if (check_bounds((c.co0 + cc) % 8 == 0 && c.co0 + cc + 32 <= a.Cout && c.w0 >= 0 && c.w0 < a.W &&
                               c.h0 + s * kTileRows + q * 4 >= 0 && c.t < a.T && c.n < a.N &&
                               sbuf + kEpiBufBytes <= epi_stage + static_cast<uint32_t>(kEpiWarps * a.epi_bufs) * kEpiBufBytes))
                tma_store_5d(&tmap_out, sbuf, c.co0 + cc, c.w0, c.h0 + s * kTileRows + q * 4, c.t, c.n);
              bulk_commit_group();
            }
            if (a.epi_bufs == 2) buf ^= 1u;
          }
        };
        uint32_t va[32], vb[32];
        // this warp's slices of the sub-tile: jj = j0, j0 + 2, ... (the two
        // warps of a quarter alternate over the tile's slices in order)
        int jj = (half + s * nsl) & 1;
        if (jj < nsl) issue(jj, va);
        while (jj < nsl) {
          tmem_ld_wait(va);
          if (jj + 2 < nsl) issue(jj + 2, vb);
          process(jj, va);
          jj += 2;
          if (jj >= nsl) break;
          tmem_ld_wait(vb);
          if (jj + 2 < nsl) issue(jj + 2, va);
          process(jj, vb);
          jj += 2;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (kPair) {
            mbar_arrive_remote(empty_leader + 8 * (accb + s));
          } else {
            mbar_arrive(acc_empty + 8 * (accb + s));
          }
        }
      }
      if (++cs == static_cast<uint32_t>(a.acc_stages)) { cs = 0; cp ^= 1; }
    }
    // the last stores must have read their staging buffers before shared memory
    // goes away; their global writes complete with the grid (a dependent launch's
    // griddepcontrol.wait covers them)
    if (!kAcc32 && lane == 0) bulk_wait_group_read<0>();
    if (!kAcc32 && a.out_amax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) out_max = max(out_max, __shfl_xor_sync(0xFFFFFFFFu, out_max, o));
      if (lane == 0) atomicMax(a.out_amax, out_max);
    }
  }

  // Reconverge every warp (one lane of warp 0 ran a role alone) before the
  // warp-aligned block / cluster barrier.
  __syncwarp();
  tc_fence_before();
  if (kPair) {
    cluster_sync();  // neither CTA leaves while its partner may still touch its memory
  } else {
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if (kPair) {
      tmem_dealloc_pair(tmem_base, a.tmem_cols);
    } else {
      tmem_dealloc(tmem_base, a.tmem_cols);
    }
  }
}

// W8A8 convolution: INT8 codes, INT32 accumulators, FP32 rescale + bias.
template <bool kAcc32, bool kPair>
__global__ void __launch_bounds__(kConvThreads, 1)
    conv3d_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_out, const ConvArgs a) {
  conv3d_body<false, kAcc32, kPair, false>(tmap_x, tmap_w, tmap_out, a);
}

// W8A8 convolution quantising its bf16 input in the kernel (scale from a maximum word).
template <bool kAcc32, bool kPair>
__global__ void __launch_bounds__(kConvThreadsFused, 1)
    conv3d_w8a8_fused_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                             const __grid_constant__ CUtensorMap tmap_out, const ConvArgs a) {
  conv3d_body<false, kAcc32, kPair, true>(tmap_x, tmap_w, tmap_out, a);
}

// Native-precision convolution: bf16 values, fp32 accumulators, + bias.
template <bool kAcc32, bool kPair>
__global__ void __launch_bounds__(kConvThreads, 1)
    conv3d_bf16_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_out, const ConvArgs a) {
  conv3d_body<true, kAcc32, kPair, false>(tmap_x, tmap_w, tmap_out, a);
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
