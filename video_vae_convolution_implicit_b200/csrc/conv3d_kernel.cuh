// conv3d_kernel.cuh -- implicit-GEMM 3D convolution for sm_100a.
//
// The convolution is the GEMM  Y[m, co] = sum_k A[m, k] * Wt[co, k]  with
//   m = ((n*Do + to)*Ho + ho)*Wo + wo   (output pixel, M = N*Do*Ho*Wo rows),
//   k = ((it*kh + ih)*kw + iw)*Cin + ci (K = kt*kh*kw*Cin, the memory order of w),
// in which A, the im2col matrix of the input, is never materialised
// (engineering.drawthings.ai, "Metal conv3d" post: conv3d computed as an
// implicit GEMM, as is usual for 2D convolution).  Padding is resolved in
// address math: spatial zero padding by the TMA im2col bounding box (out of
// range pixels read as zero), temporal padding by choosing, per tile and
// temporal tap, which source frame the TMA reads (frame 0 again for causal
// replicate padding; the tap is skipped when it reads zero padding), so no
// padded copy of the input is ever written.
//
// One CTA per SM, persistent over output tiles of 128 pixels x BN output
// channels (or a CTA pair over 256-pixel tiles, or the transposed product
// for layers with at most 128 output channels: see the kernel).  Warp roles
// (192 threads):
//   warp 0     TMA producer: per k-block one im2col load of A (128 pixels x 64
//              channels of one tap) and one tiled load of B (BN x 64), both
//              128-byte swizzled, into a ring of `stages` shared-memory slots
//              guarded by full/empty mbarriers;
//   warp 1     allocates tensor memory and issues tcgen05.mma (M=128, N=BN,
//              K=16, four per k-block) into one of two fp32 TMEM accumulators;
//   warps 2-5  epilogue: tcgen05.ld, + bias, + residual (fetched ahead by
//              TMA), one rounding to the output type (or fp32 output for the
//              backward pass's padded frames), staged through swizzled shared
//              memory and written by TMA stores; then frees the accumulator so
//              the next tile's main loop overlaps this tile's epilogue.
// Every mbarrier wait is bounded in time; a wait that runs out records
// CONV3D_ERR_TIMEOUT in the status word, and all roles leave their loops,
// drain their asynchronous work and free tensor memory before exiting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace conv3d {

constexpr int BM = 128;             // output pixels per tile (TMEM lanes)
constexpr int BK = 64;              // channels per k-block (128 bytes of fp16/bf16)
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;

// Optional parts of the forward kernel, compiled into the instances that use
// them only, so the plain convolution keeps a compact epilogue (measured: with
// these paths behind run-time flags in one instance the 1x1x1 layer, whose
// epilogue runs every 8 k-blocks, slowed from 159 to 260 us).
constexpr int FEAT_SPLIT = 1;      // tail split: K pieces, partials, tickets
constexpr int FEAT_STATS = 2;      // GroupNorm statistics of the output
constexpr int FEAT_SCATTER = 4;    // strided output (data-gradient phases)
constexpr int FEAT_GN = 8;         // GroupNorm + SiLU of the x operand (4 more warps)
constexpr int FEAT_LO8 = 16;       // first frame: the lo weight product in e5m2 (kind::f8f6f4)
constexpr int FEAT_MIXED = 32;     // fp32 front frames and 16-bit frames in one launch (data gradient)
constexpr int FEAT_COMBINE = 64;   // output frame 0 also sums the kt-1 virtual frames before it
constexpr int FEAT_EPI8 = 128;     // 8 epilogue warps, two per TMEM lane quarter (short-K launches)
constexpr int BK8 = 128;           // 8-bit channels per k-block (128-byte rows, like BK 16-bit ones)
constexpr int GN_THREADS = 320;     // with the GroupNorm + SiLU operand transform (4 more warps)
constexpr int EPI8_THREADS = 320;   // with 8 epilogue warps
constexpr int MAX_STAGES = 8;

constexpr int STATUS_TIMEOUT = 5;   // mirrors CONV3D_ERR_TIMEOUT

struct KernelParams {
  int D, Do, Ho, Wo;                 // input frames; output extents
  int H, W;                          // input extents
  int HoWo;
  int Cin, Cout;
  int kt, kh, kw;
  int pf, ph, pw;                    // front temporal pad, spatial pads
  int st, sh, sw;                    // strides
  int tpad;                          // 0 zero, 1 causal replicate, 2 causal zero, 3 cached
  int n_chunks;                      // ceil(Cin / BK)
  // First frame with the lo product in 8 bits (FEAT_LO8): temporal tap 1 of
  // the folded (hi, lo) pair runs n_chunks8 = ceil(Cin / BK8) k-blocks per
  // spatial tap of e5m2 operands -- x * 2^-8 through map_p (im2col, 128
  // channels a box) and lo * 2^8 through map_f ([Cout][kh*kw][Cin]) -- with
  // tcgen05.mma kind::f8f6f4 and instruction descriptor idesc8; the scales
  // cancel in the product, which adds into the same fp32 accumulator.
  // n_chunks8 = 0 otherwise.
  int n_chunks8;
  uint32_t idesc8;
  int BN;                            // MMA N: channels per tile, or 256 pixels (swapped)
  int co_tile;                       // output channels per tile
  int pix_tile;                      // output pixels per tile (128, or 256 for a CTA pair / swapped)
  int n_tiles_n;                     // ceil(Cout / co_tile)
  int tiles_per_frame;               // ceil(HoWo / pix_tile)
  int num_tiles;
  // Tail split: tiles [split_first, num_tiles) are each cut into split_s
  // pieces along K, so that the work of the last, partly filled round of
  // tiles spreads over every SM.  Work items: split_s consecutive pieces per
  // split tile first, then tiles 0 .. split_first-1 whole (num_items in all).
  // The pieces run in the first round, so the epilogue that adds up their
  // partials overlaps the whole tiles' main loops instead of ending the launch.
  int num_items;
  int split_first;
  int split_s;                       // 1: no tail split
  float* part;                       // [tail tiles][split_s][128 lanes][BN] fp32 partials
  unsigned long long* ticket;        // [tail tiles][4 lane quarters]: (generation << 32) |
                                     // pieces whose partial is stored
  unsigned int gen;                  // this launch's generation (nonzero)
  int stages;
  uint32_t tmem_cols;                // power of two >= 2*BN
  uint32_t idesc;
  const void* bias;                  // [Cout] or null
  int has_residual;                  // residual is read through map_r
  int out_f32;                       // y is fp32 (one-CTA variants)
  // Mixed output (the data gradient under causal replicate padding): the
  // first f32_frames output frames of each sample are the fp32 parts of dx
  // frame 0 and go through map_f (N * f32_frames frames); output frame
  // to >= f32_frames is dx frame to - f32_frames + 1, 16-bit, through map_y
  // (N * y_frames frames).  0: every frame through map_y.
  int f32_frames;
  int y_frames;
  // Combined front (the data gradient under causal replicate padding,
  // FEAT_COMBINE): the tiles of output frame 0 also run the taps of the kt-1
  // virtual frames -1 .. -(kt-1) before it, all into one accumulator, so that
  // frame 0 gets the gradient of its replicated copies with one rounding.
  // 0: off (kt when on).
  int combine;
  int* status;                       // device status word
  unsigned long long timeout_ns;
  int test_stall;                    // failure-detection test: the producer skips the
                                     // copies of its first stage (armed from the host)
  // GroupNorm + SiLU applied to x as the kernel reads it (GroupNorm variant):
  // h = silu((x - mean) * rstd * gamma + beta) per statistic set and group
  const double* gn_stats;            // [sets][groups][2] {mean, rstd}
  const uint16_t* gn_gamma;          // [Cin] or null (1)
  const uint16_t* gn_beta;           // [Cin] or null (0)
  int gn_groups;
  int gn_per_frame;                  // sets are frames of a sample (else whole samples)
  int gn_silu;                       // apply the SiLU after the normalisation
  // GroupNorm statistics of y (per sample) gathered by the epilogue from the
  // rounded outputs: fp64 {sum, sum of squares} added into gn_out
  // [N][gn_out_groups][2] (zeroed by the host), or null
  double* gn_out;
  int gn_out_groups;                 // at most 64; divides Cout
  // Strided output (one phase of the data gradient of a strided convolution):
  // output pixel (a, b) of output frame f is element
  // [f][a*sc_sh + sc_rh][b*sc_sw + sc_rw] of y_scatter, frames sc_H x sc_W,
  // written by plain stores from registers instead of the TMA store map
  // (16-bit outputs, no residual); null otherwise.
  uint16_t* y_scatter;
  int sc_sh, sc_sw, sc_rh, sc_rw, sc_H, sc_W;
};

// Epilogue staging: each epilogue warp owns two 32-row x 32-channel buffers
// (64-byte rows, 64-byte swizzle) for y and, with a residual, two more.
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF_BYTES = 32 * 32 * 2;
constexpr int EPI_Y_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;

// Byte offset of 16-byte chunk c of row r in a 32 x 64-byte buffer written or
// read by TMA with the 64-byte swizzle (chunk index XOR bits 7-8 of the row
// offset).
__device__ __forceinline__ uint32_t swz64(uint32_t r, uint32_t c) {
  return r * 64u + ((c ^ ((r >> 1) & 3u)) << 4);
}

// The same for 32 x 128-byte rows (fp32 output) with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz128(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

struct Tile {
  int frame_out;  // n*Do + to
  int n, to;
  int p0;         // first output pixel of the tile inside its frame
  int co0;
};

__device__ __forceinline__ Tile decode_tile(const KernelParams& p, int t) {
  Tile r;
  const int nt = t % p.n_tiles_n;
  const int mt = t / p.n_tiles_n;
  r.frame_out = mt / p.tiles_per_frame;
  r.p0 = (mt - r.frame_out * p.tiles_per_frame) * p.pix_tile;
  r.n = r.frame_out / p.Do;
  r.to = r.frame_out - r.n * p.Do;
  r.co0 = nt * p.co_tile;
  return r;
}

// One work item: a whole tile, or one K-range piece of a tail tile.
struct Work {
  Tile tl;
  int kb_lo, kb_hi;  // the item's k-blocks, in the tile's k-block order
  int slot;          // partial slot (tail tile * split_s + piece), or -1 for a whole tile
};

__device__ __forceinline__ int kblocks_of_tile(const KernelParams& p, int to);

template <bool kSplit>
__device__ __forceinline__ Work decode_work(const KernelParams& p, int i) {
  Work w;
  int t = i, piece = -1;
  if (kSplit) {
    const int pieces = (p.num_tiles - p.split_first) * p.split_s;
    if (i < pieces) {
      const int q = i / p.split_s;
      t = p.split_first + q;
      piece = i - q * p.split_s;
    } else {
      t = i - pieces;
    }
  }
  w.tl = decode_tile(p, t);
  const int nkb = kblocks_of_tile(p, w.tl.to);
  if (piece < 0) {
    w.kb_lo = 0;
    w.kb_hi = nkb;
    w.slot = -1;
  } else {
    w.kb_lo = piece * nkb / p.split_s;
    w.kb_hi = (piece + 1) * nkb / p.split_s;
    w.slot = (t - p.split_first) * p.split_s + piece;
  }
  return w;
}

constexpr int kNoFrame = -0x40000000;

// Source frame read by temporal tap `it` of output frame `to`: a frame of x
// (>= 0), a cached frame of the previous chunk (-(kt-1) .. -1, cached mode), or
// kNoFrame when the tap reads zero padding (and contributes nothing).
__device__ __forceinline__ int source_frame(const KernelParams& p, int to, int it) {
  const int f = to * p.st + it - p.pf;
  if (f < 0) {
    if (p.tpad == 1) return 0;      // causal replicate: frame 0
    if (p.tpad == 3) return f;      // cached frame kt-1+f of the previous chunk
    return kNoFrame;                // zero padding
  }
  return f < p.D ? f : kNoFrame;
}

__device__ __forceinline__ int kblocks_of_tile(const KernelParams& p, int to) {
  int valid = 0;
  const int nv = p.combine > 0 && to == 0 ? p.combine : 1;   // frame 0 and the frames before it
  for (int v = 0; v < nv; ++v)
    for (int it = 0; it < p.kt; ++it) valid += source_frame(p, to - v, it) != kNoFrame;
  if (p.n_chunks8 > 0) return p.kh * p.kw * (p.n_chunks + p.n_chunks8);   // folded hi + e5m2 lo
  return valid * p.kh * p.kw * p.n_chunks;
}

struct SharedCtl {
  volatile int* abort_flag;
  int* status;
  unsigned long long timeout_ns;
  uint32_t peer_abort;   // shared::cluster address of the peer CTA's abort flag (pairs), or 0
};

// Every role of this CTA (and of its peer, for a pair) leaves its loop.
__device__ __forceinline__ void raise_abort(const SharedCtl& c, int code) {
  *c.abort_flag = 1;
  if (c.peer_abort != 0) st_cluster_u32(c.peer_abort, 1);
  atomicCAS(c.status, 0, code);
}

// Wait for the phase of `bar` with the given parity.  Returns false when the
// wait ran out of time (and then raises the abort) or, if `watch_abort`, when
// another role already aborted.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const SharedCtl& c,
                                          bool watch_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15) == 0) {
      if (watch_abort && *c.abort_flag) return false;
      if (globaltimer_ns() - t0 > c.timeout_ns) {
        raise_abort(c, STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

// The same for a barrier that the peer CTA of a pair arrives on with release
// semantics at cluster scope (what it stored before arriving is then visible).
__device__ __noinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity,
                                                  const SharedCtl& c) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 15) == 15 && globaltimer_ns() - t0 > c.timeout_ns) {
      raise_abort(c, STATUS_TIMEOUT);
      return false;
    }
  }
}

// End of a producer's loop.  After an abort no copy may still be writing into
// shared memory when the CTA exits, so the producer waits until every stage
// instance it (and, for a CTA pair, its peer) announced has landed:
//   issued      stage instances this producer counted; with `skip_first`
//               (the failure-detection test) instance 0 was counted but
//               neither announced nor copied;
//   half_bytes  one CTA's share of a stage's bytes (pairs).
// The copies of both CTAs of a pair complete on the even CTA's barriers, so
// the odd CTA publishes its own count in the even CTA (`peer_count`, a
// release-arrive on `peer_bar`) at the end of every run, and the even CTA
// settles each instance that only one of the two issued before waiting on it:
// an instance it announced whose odd half will never come has that half
// cancelled (complete_tx); one whose odd half is in flight but which it never
// announced is announced now for that half alone.  Both producers are paced
// by the same empty barriers and the MMAs need both halves, so the counts
// differ by at most `stages` and every instance before max - stages has been
// consumed.
template <bool kPair>
__device__ void producer_finish(bool aborted, long long issued, bool skip_first, int stages,
                                uint32_t full_bar, uint32_t half_bytes, uint32_t peer_count,
                                uint32_t peer_bar, const SharedCtl& c, bool leader) {
  if constexpr (kPair) {
    if (!leader) {
      st_cluster_u64(mapa_shared(peer_count, 0), static_cast<unsigned long long>(issued));
      mbar_arrive_cluster(mapa_shared(peer_bar, 0));
      return;
    }
  }
  if (!aborted) return;
  long long peer = issued;
  if constexpr (kPair) {
    if (!wait_bounded_cluster(peer_bar, 0, c)) return;   // the peer never reported
    unsigned long long v;
    asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(peer_count) : "memory");
    peer = static_cast<long long>(v);
  }
  const long long top = issued > peer ? issued : peer;
  const long long first = top > stages ? top - stages : 0;
  for (long long i = first; i < top; ++i) {
    if (skip_first && i == 0) continue;
    const uint32_t fb = full_bar + 8 * static_cast<uint32_t>(i % stages);
    if constexpr (kPair) {
      if (i < issued && i >= peer) mbar_complete_tx(fb, half_bytes);
      else if (i >= issued && i < peer) mbar_arrive_expect_tx(fb, half_bytes);
    }
    wait_bounded(fb, static_cast<uint32_t>((i / stages) & 1), c, false);
  }
}

// Ticket of one lane quarter of a split tail tile: counts, for this launch's
// generation, the pieces whose partial is stored (a count of another
// generation -- left by a launch that aborted -- counts as none).  True for
// the piece that completes the quarter, which also resets the ticket to 0: no
// other piece of the launch touches it afterwards, so a launch that runs again
// with the same parameters (a CUDA graph replay) starts from zero.  Each
// retry means another piece got in first, so at most split_s attempts.
__device__ __forceinline__ bool take_ticket(unsigned long long* t, unsigned int gen, int pieces) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(t);
  for (;;) {
    const unsigned long long done = (cur >> 32) == gen ? (cur & 0xFFFFFFFFull) : 0ull;
    const unsigned long long next = (static_cast<unsigned long long>(gen) << 32) | (done + 1);
    const unsigned long long seen = atomicCAS(t, cur, next);
    if (seen == cur) {
      const bool last = done + 1 == static_cast<unsigned long long>(pieces);
      if (last) atomicExch(t, 0ull);
      return last;
    }
    cur = seen;
  }
}

// A slot holds a 128-lane x BN-column fp32 accumulator as float4 groups
// [column chunk j][group q of 4 columns][lane]: lane l's columns 32j + 4q ..
// +3 are float4 number (j*8 + q)*128 + l, so each warp access covers 32
// consecutive float4 (512 contiguous bytes).
__device__ __forceinline__ float4* slot_at(const KernelParams& p, int slot) {
  return reinterpret_cast<float4*>(p.part) + static_cast<size_t>(slot) * (BM / 4) * p.BN;
}

// Tail piece, for the calling warp's 32 TMEM lanes (lane row = quarter*32 +
// lane) and its 32-column chunks j0, j0 + jstep, ...: store the raw fp32
// accumulator in the piece's slot, then take the ticket of epilogue warp ew
// (8 per tail tile).  Returns true in every lane of the warp whose piece
// completed these lanes and chunks; every piece's partial of them is then
// visible to the warp.  Warp-level only (no other warp is
// waited for), so an abort in another warp cannot hold this one.
__device__ __forceinline__ bool store_piece(const KernelParams& p, int slot, uint32_t t_row,
                                            bool has_acc, uint32_t quarter, uint32_t lane,
                                            int j0, int jstep, uint32_t ew) {
  float4* dst = slot_at(p, slot) + quarter * 32u + lane;
  for (int j = j0; j < p.BN / 32; j += jstep) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(t_row + j * 32, r);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 8; ++q)
      dst[(j * 8 + q) * BM] =
          has_acc ? make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]))
                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0)
    last = take_ticket(p.ticket + (slot / p.split_s) * 8 + ew, p.gen, p.split_s) ? 1 : 0;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (last) __threadfence();
  return last != 0;
}

// Columns [32j, 32j+32) of the calling lane's row of a completed tail tile:
// the sum of every piece's partial, in piece order (the result does not
// depend on which piece finished last).  L2 loads: the partials were written
// by other SMs.
__device__ __forceinline__ void sum_pieces(const KernelParams& p, int slot0, uint32_t lane_row,
                                           int j, float (&v)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = 0.0f;
  for (int sp = 0; sp < p.split_s; ++sp) {
    const float4* src = slot_at(p, slot0 + sp) + j * 8 * BM + lane_row;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 a = __ldcg(src + q * BM);
      v[4 * q] += a.x;
      v[4 * q + 1] += a.y;
      v[4 * q + 2] += a.z;
      v[4 * q + 3] += a.w;
    }
  }
}

// silu(z) = z * sigmoid(z) = h + h * tanh(h) with h = z/2: one special-function
// operation (the hardware tanh approximation, relative error about 2^-11,
// below the 2^-9 of the rounding that follows).
__device__ __forceinline__ float silu_fast(float z) {
  const float h = 0.5f * z;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

// Output GroupNorm statistics, gathered by each epilogue warp for the
// channels it meets: lane l keeps fp64 {sum, sum of squares} of channel
// base + 32k + l for every 32-channel window k of the current tiles (the
// single variant: a tile's BN channels, one window per 32-channel chunk; the
// transposed variant: the warp's own 32 channels, one window).  A chunk adds
// its fp32 partial (at most 32 values); the windows are reduced to their
// groups and added to the global sums only when the sample or the channel
// base changes, and at the end.
struct GnAcc {
  double s[8], q[8];
  int n, co0;   // sample and channel base being gathered (n < 0: none)
};

// Adds the warp's sums of window k (channels c0 + lane) to the global sums of
// their groups, then clears them.
__device__ __forceinline__ void gn_flush_window(double* dst, int Cout, int cg, int c0, double& s,
                                                double& q, uint32_t lane) {
  const int c = c0 + static_cast<int>(lane);
  const int my_g = c < Cout ? c / cg : -1;
  const int g_last = (c0 + 31 < Cout ? c0 + 31 : Cout - 1) / cg;
  for (int g = c0 / cg; g <= g_last; ++g) {
    double ts = my_g == g ? s : 0.0, tq = my_g == g ? q : 0.0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ts += __shfl_xor_sync(0xFFFFFFFFu, ts, off);
      tq += __shfl_xor_sync(0xFFFFFFFFu, tq, off);
    }
    if (lane == 0) {
      atomicAdd(dst + 2 * g, ts);
      atomicAdd(dst + 2 * g + 1, tq);
    }
  }
  s = q = 0.0;
}

// Flushes every window of the accumulator (windows of 32 channels from a.co0,
// or from a.co0 + base_off for the transposed variant's one window).
__device__ __forceinline__ void gn_flush(double* gn_out, int groups, int Cout, GnAcc& a,
                                         int windows, int base_off, uint32_t lane) {
  if (a.n >= 0) {
    double* dst = gn_out + static_cast<size_t>(a.n) * groups * 2;
    const int cg = Cout / groups;
    for (int k = 0; k < windows; ++k) {
      const int c0 = a.co0 + base_off + 32 * k;
      if (c0 < Cout) gn_flush_window(dst, Cout, cg, c0, a.s[k], a.q[k], lane);
    }
  }
}

template <bool kBF16>
struct Cvt;

template <>
struct Cvt<true> {
  static __device__ __forceinline__ float lo(uint32_t v) { return __uint_as_float(v << 16); }
  static __device__ __forceinline__ float hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <>
struct Cvt<false> {
  static __device__ __forceinline__ float lo(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
  }
  static __device__ __forceinline__ float hi(uint32_t v) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
  }
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

// Two floats to two e5m2 bytes (first in the low byte), round to nearest,
// saturating to the largest finite value.
__device__ __forceinline__ uint32_t e5m2x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E5M2));
}

// kPair = false: one CTA per tile of 128 pixels x BN channels (cta_group::1).
// kPair = true:  a cluster of two CTAs per tile of 256 pixels x BN channels
//   (cta_group::2, M = 256): CTA r loads the A rows [128r, 128r+128) of the
//   tile and the B rows [BN/2 r, BN/2 (r+1)) into its own shared memory, both
//   loads signalling the even CTA's full barrier; the even CTA issues the MMAs
//   and commits them to the stage and accumulator barriers of both CTAs; each
//   CTA's epilogue drains its own TMEM (its 128 rows) and releases the
//   accumulator on the even CTA's barrier.  No load is shared between the CTAs.
// kSwap = true (one CTA): the transposed product Y^T = W * A^T, so that layers
//   with few output channels still issue full-width MMAs: M = 128 output
//   channels (the weight tile is the A operand), N = 256 output pixels (the
//   im2col tile is the B operand).  TMEM lane = channel, column = pixel; the
//   epilogue transposes through shared memory before the TMA store.
// kGN (single-CTA and transposed variants): four more warps (6-9) apply
//   GroupNorm + SiLU to the x operand in shared memory between its TMA load
//   and the MMAs that read it, so that the normalised activation is never
//   written to memory: rows that hold spatial padding stay zero (the padding
//   belongs to the normalised tensor), and the tensor-core issuer waits for
//   the transform of a stage instead of its load.
template <bool kBF16, bool kPair, bool kSwap, int kFeat = 0>
__global__ void __launch_bounds__((kFeat & FEAT_GN)     ? GN_THREADS
                                  : (kFeat & FEAT_EPI8) ? EPI8_THREADS
                                                        : NUM_THREADS,
                                  1)
    conv3d_implicit_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                const __grid_constant__ CUtensorMap map_b,
                                const __grid_constant__ CUtensorMap map_y,
                                const __grid_constant__ CUtensorMap map_r,
                                const __grid_constant__ CUtensorMap map_p,
                                const __grid_constant__ CUtensorMap map_f,
                                const KernelParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ __align__(8) uint64_t s_peer_bar;      // pairs: the odd CTA's end-of-run report
  __shared__ unsigned long long s_peer_count;

  constexpr bool kSplit = (kFeat & FEAT_SPLIT) != 0;
  constexpr bool kStats = (kFeat & FEAT_STATS) != 0;
  constexpr bool kScatter = (kFeat & FEAT_SCATTER) != 0;
  constexpr bool kGN = (kFeat & FEAT_GN) != 0;
  constexpr bool kLo8 = (kFeat & FEAT_LO8) != 0;
  constexpr bool kMixed = (kFeat & FEAT_MIXED) != 0;
  constexpr bool kComb = (kFeat & FEAT_COMBINE) != 0;
  constexpr bool kEpi8 = (kFeat & FEAT_EPI8) != 0;
  constexpr int kYBufs = 2;   // output staging buffers per epilogue warp
  // With 8 epilogue warps, warps q and q+4 of the epilogue share TMEM lane
  // quarter q and take its even and odd 32-column chunks.
  constexpr int kEpiWarps = kEpi8 ? 2 * EPI_WARPS : EPI_WARPS;
  constexpr int kJStep = kEpi8 ? 2 : 1;
  static_assert(!(kEpi8 && (kPair || kGN || kStats || kScatter || kLo8 || kMixed || kComb)),
                "8 epilogue warps: one CTA, plain output (optionally split)");
  static_assert(!(kLo8 && (kPair || kSwap)), "the e5m2 lo product: one CTA, M = pixels");
  constexpr int kCtas = kPair ? 2 : 1;
  const uint32_t warp = threadIdx.x / 32;
  const uint32_t lane = threadIdx.x % 32;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int unit = blockIdx.x / kCtas;        // this CTA's cluster (or CTA) index
  const int num_units = gridDim.x / kCtas;

  // Carve shared memory: A ring, B ring (both 1024-byte aligned for the
  // 128-byte swizzle), then the mbarriers.
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t b_rows = static_cast<uint32_t>(p.BN) / kCtas;
  const uint32_t b_stage_bytes = b_rows * BK * 2;
  const uint32_t a_ring = base;
  const uint32_t b_ring = a_ring + p.stages * A_STAGE_BYTES;
  const uint32_t ybytes =
      (p.out_f32 || p.f32_frames > 0) ? 2 * EPI_BUF_BYTES : EPI_BUF_BYTES;   // one y buffer
  const uint32_t y_stage = b_ring + p.stages * b_stage_bytes;        // [kEpiWarps][2] buffers
  const uint32_t r_stage = y_stage + kEpiWarps * kYBufs * ybytes;     // 2 per warp, with a residual
  const uint32_t bars = r_stage + (p.has_residual ? kEpiWarps * 2 * EPI_BUF_BYTES : 0);
  const uint32_t full_bar = bars;                         // [stages]
  const uint32_t empty_bar = bars + 8 * p.stages;         // [stages]
  const uint32_t tfull_bar = bars + 16 * p.stages;        // [2]
  const uint32_t tempty_bar = tfull_bar + 16;             // [2]
  const uint32_t drain_bar = tempty_bar + 16;             // [1]
  const uint32_t rfull_bar = drain_bar + 8;               // [kEpiWarps][2]
  const uint32_t ready_bar = rfull_bar + 16 * kEpiWarps;  // [stages] (GroupNorm variant)

  SharedCtl ctl{&s_abort, p.status, p.timeout_ns,
                kPair ? mapa_shared(smem_addr(&s_abort), rank ^ 1u) : 0u};
  const uint32_t peer_bar = smem_addr(&s_peer_bar);
  const uint32_t peer_count = smem_addr(&s_peer_count);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar + 8 * a, 1);
      mbar_init(tempty_bar + 8 * a, kEpiWarps * kCtas);
    }
    mbar_init(drain_bar, 1);
    mbar_init(peer_bar, 1);
    for (int e = 0; e < 2 * kEpiWarps; ++e) mbar_init(rfull_bar + 8 * e, 1);
    if constexpr (kGN)
      for (int s = 0; s < p.stages; ++s) mbar_init(ready_bar + 8 * s, 4);
    fence_mbar_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_y);
    if (p.has_residual) prefetch_tensormap(&map_r);
    if (p.tpad == 3) prefetch_tensormap(&map_p);
    if (p.f32_frames > 0) prefetch_tensormap(&map_f);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_addr(&s_tmem_base), p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(&s_tmem_base), p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();   // the peer's barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  // Launched as a programmatic dependent of the previous kernel on the stream
  // (which may still be running): everything above touched only this CTA's
  // own resources; no global memory is read or written before this point.
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t tx_bytes = kCtas * (A_STAGE_BYTES + b_stage_bytes);
      const bool stall = p.test_stall != 0;
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int i = unit; ok && i < p.num_items; i += num_units) {
        const Work wk = decode_work<kSplit>(p, i);
        const Tile& tl = wk.tl;
        int kb = 0;          // k-block index within the tile; the item issues [kb_lo, kb_hi)
        const int kb_hi = kSplit ? wk.kb_hi : 0x7FFFFFFF;   // whole tiles: no bound to test
        // first output pixel of this CTA's rows; rows past the frame are
        // computed from any valid window origin and masked by the epilogue
        int row0 = tl.p0 + static_cast<int>(rank) * BM;
        if (row0 >= p.HoWo) row0 = 0;
        const int ho0 = row0 / p.Wo;
        const int wo0 = row0 - ho0 * p.Wo;
        const int w_org = wo0 * p.sw - p.pw;   // window origin of the first pixel
        const int h_org = ho0 * p.sh - p.ph;
        const int co_b = tl.co0 + static_cast<int>(rank * b_rows);
        // kComb: frame 0's tiles also take the taps of the virtual frames before it
        const int nvt = (kComb && tl.to == 0 ? p.combine : 1) * p.kt;
        for (int vt = 0; ok && kb < kb_hi && vt < nvt; ++vt) {
          const int it = kComb ? vt % p.kt : vt;
          const int f = source_frame(p, kComb ? tl.to - vt / p.kt : tl.to, it);
          if (f == kNoFrame) continue;
          // frames before the chunk come from the cached-frames tensor
          const CUtensorMap* xmap = f < 0 ? &map_p : &map_a;
          const int img = f < 0 ? tl.n * (p.kt - 1) + (p.kt - 1) + f : tl.n * p.D + f;
          for (int ih = 0; ok && kb < kb_hi && ih < p.kh; ++ih) {
            for (int iw = 0; ok && kb < kb_hi && iw < p.kw; ++iw) {
              const int tap = (it * p.kh + ih) * p.kw + iw;
              const bool lo8 = kLo8 && it == 1;   // the e5m2 lo product
              const int nch = lo8 ? p.n_chunks8 : p.n_chunks;
              for (int cc = 0; cc < nch && kb < kb_hi; ++cc) {
                if (kSplit && kb++ < wk.kb_lo) continue;   // an earlier piece's k-block
                if (!wait_bounded(empty_bar + 8 * stage, phase ^ 1, ctl, true)) {
                  ok = false;
                  break;
                }
                const uint32_t fb = full_bar + 8 * stage;
                if (stall && issued == 0) {
                  // failure-detection test: this stage never fills, so the
                  // tensor-core issuer's wait on it must run out
                } else if constexpr (kSwap) {
                  // A operand = 128 output channels of w, B operand = 256 pixels
                  mbar_arrive_expect_tx(fb, tx_bytes);
                  tma_load_3d(a_ring + stage * A_STAGE_BYTES, &map_b, fb, cc * BK, tap, tl.co0);
                  tma_load_im2col_4d(b_ring + stage * b_stage_bytes, xmap, fb, cc * BK, w_org,
                                     h_org, img, static_cast<uint16_t>(iw),
                                     static_cast<uint16_t>(ih));
                } else if constexpr (kPair) {
                  if (leader) mbar_arrive_expect_tx(fb, tx_bytes);
                  const uint32_t fb_leader = mapa_shared(fb, 0);
                  tma_load_im2col_4d_pair(a_ring + stage * A_STAGE_BYTES, xmap, fb_leader,
                                          cc * BK, w_org, h_org, img, static_cast<uint16_t>(iw),
                                          static_cast<uint16_t>(ih));
                  tma_load_3d_pair(b_ring + stage * b_stage_bytes, &map_b, fb_leader, cc * BK,
                                   tap, co_b);
                } else if (lo8) {
                  // same bytes as a 16-bit k-block: 128-byte rows of 128 channels
                  mbar_arrive_expect_tx(fb, tx_bytes);
                  tma_load_im2col_4d(a_ring + stage * A_STAGE_BYTES, &map_p, fb, cc * BK8, w_org,
                                     h_org, img, static_cast<uint16_t>(iw),
                                     static_cast<uint16_t>(ih));
                  tma_load_3d(b_ring + stage * b_stage_bytes, &map_f, fb, cc * BK8,
                              ih * p.kw + iw, co_b);
                } else {
                  mbar_arrive_expect_tx(fb, tx_bytes);
                  tma_load_im2col_4d(a_ring + stage * A_STAGE_BYTES, xmap, fb, cc * BK, w_org,
                                     h_org, img, static_cast<uint16_t>(iw),
                                     static_cast<uint16_t>(ih));
                  tma_load_3d(b_ring + stage * b_stage_bytes, &map_b, fb, cc * BK, tap, co_b);
                }
                ++issued;
                if (++stage == static_cast<uint32_t>(p.stages)) {
                  stage = 0;
                  phase ^= 1;
                }
              }
            }
          }
        }
      }
      producer_finish<kPair>(!ok, issued, stall, p.stages, full_bar, A_STAGE_BYTES + b_stage_bytes,
                             peer_count, peer_bar, ctl, leader);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int local = 0;
      for (int i = unit; ok && i < p.num_items; i += num_units, ++local) {
        const Work wk = decode_work<kSplit>(p, i);
        const int nkb = wk.kb_hi - wk.kb_lo;
        const uint32_t acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!wait_bounded(tempty_bar + 8 * acc, acc_phase ^ 1, ctl, true)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(p.BN);
        for (int kb = 0; kb < nkb; ++kb) {
          // the stage's copies have landed (and, GroupNorm variant, been transformed)
          if (!wait_bounded((kGN ? ready_bar : full_bar) + 8 * stage, phase, ctl, true)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc_k_sw128(a_ring + stage * A_STAGE_BYTES);
          const uint64_t db = smem_desc_k_sw128(b_ring + stage * b_stage_bytes);
          // the e5m2 lo k-blocks follow the kh*kw*n_chunks hi ones in a tile
          const bool lo8 = kLo8 && wk.kb_lo + kb >= p.kh * p.kw * p.n_chunks;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // +32 bytes along K inside the swizzled 128-byte row = +2 in the
            // descriptor's address field (16 16-bit or 32 8-bit values).
            if constexpr (kPair)
              mma_f16_ss_pair(d_tmem, da + 2 * k, db + 2 * k, p.idesc, (kb | k) != 0);
            else if (lo8)
              mma_f8_ss(d_tmem, da + 2 * k, db + 2 * k, p.idesc8, (kb | k) != 0);
            else
              mma_f16_ss(d_tmem, da + 2 * k, db + 2 * k, p.idesc, (kb | k) != 0);
          }
          if constexpr (kPair) {
            mma_commit_pair(empty_bar + 8 * stage);
            mma_commit_pair(mapa_shared(empty_bar + 8 * stage, 1));
          } else {
            mma_commit(empty_bar + 8 * stage);
          }
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (kPair) {
          mma_commit_pair(tfull_bar + 8 * acc);
          mma_commit_pair(mapa_shared(tfull_bar + 8 * acc, 1));
        } else {
          mma_commit(tfull_bar + 8 * acc);
        }
      }
      // All tensor-core work of this CTA (pair) has finished once the drain fires.
      if constexpr (kPair)
        mma_commit_pair(drain_bar);
      else
        mma_commit(drain_bar);
      wait_bounded(drain_bar, 0, ctl, false);
    }
  } else if (kGN && warp >= 2 + EPI_WARPS) {
    // ------------------------------------------------------------ GroupNorm + SiLU of x
    // The x operand of a stage is `rows` rows (output pixels) of 64 channels,
    // 128 bytes each, 128-byte swizzled: 16-byte chunk c of row r sits at
    // physical chunk c ^ (r & 7).  Thread t owns physical chunk t & 7 of the
    // rows t/8 + 16j, whose low three bits are all those of t/8, so it always
    // sees the same logical chunk: channels 8 * ((t & 7) ^ (t/8 & 7)) .. +7 of
    // the k-block, whose scale and shift it keeps in registers.  Rows whose
    // window position is spatial padding were zero-filled by the TMA and stay
    // zero; the others become h = silu(x * scale + shift) rounded once.
    using C = Cvt<kBF16>;
    constexpr int kRows = kSwap ? 16 : 8;         // 256 or 128 rows per operand stage
    const uint32_t t = threadIdx.x - 32u * (2 + EPI_WARPS);
    const uint32_t pchunk = t & 7u;
    const uint32_t r0 = t >> 3;
    const uint32_t lchunk = pchunk ^ (r0 & 7u);
    const uint32_t x_ring = kSwap ? b_ring : a_ring;
    const uint32_t x_stage = kSwap ? b_stage_bytes : static_cast<uint32_t>(A_STAGE_BYTES);
    const int cg = p.Cin / p.gn_groups;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int i = unit; ok && i < p.num_items; i += num_units) {
      const Work wk = decode_work<kSplit>(p, i);
      const Tile& tl = wk.tl;
      // output pixel of each of this thread's rows (ho < 0: past the frame)
      int rho[kRows], rwo[kRows];
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        const int q = tl.p0 + static_cast<int>(r0) + 16 * j;
        rho[j] = q < p.HoWo ? q / p.Wo : -0x100000;
        rwo[j] = q < p.HoWo ? q - rho[j] * p.Wo : 0;
      }
      int kb = 0;
      for (int it = 0; ok && kb < wk.kb_hi && it < p.kt; ++it) {
        const int f = source_frame(p, tl.to, it);
        if (f == kNoFrame) continue;
        const int set = p.gn_per_frame ? tl.n * p.D + f : tl.n;
        const double* st = p.gn_stats + static_cast<size_t>(set) * p.gn_groups * 2;
        for (int ih = 0; ok && kb < wk.kb_hi && ih < p.kh; ++ih) {
          for (int iw = 0; ok && kb < wk.kb_hi && iw < p.kw; ++iw) {
            for (int cc = 0; cc < p.n_chunks && kb < wk.kb_hi; ++cc) {
              if (kb++ < wk.kb_lo) continue;
              if (!wait_bounded(full_bar + 8 * stage, phase, ctl, true)) {
                ok = false;
                break;
              }
              const int c0 = cc * BK + static_cast<int>(lchunk) * 8;
              if (c0 < p.Cin) {          // channels past Cin meet zero weights
                float sc[8], sh[8];
                uint4 ga = make_uint4(0, 0, 0, 0), be = make_uint4(0, 0, 0, 0);
                if (p.gn_gamma) ga = __ldg(reinterpret_cast<const uint4*>(p.gn_gamma + c0));
                if (p.gn_beta) be = __ldg(reinterpret_cast<const uint4*>(p.gn_beta + c0));
                const uint32_t gw[4] = {ga.x, ga.y, ga.z, ga.w};
                const uint32_t bw[4] = {be.x, be.y, be.z, be.w};
                int g_prev = -1;
                float mean = 0.0f, rstd = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const int g = (c0 + e) / cg;
                  if (g != g_prev) {
                    mean = static_cast<float>(st[2 * g]);
                    rstd = static_cast<float>(st[2 * g + 1]);
                    g_prev = g;
                  }
                  const float gam = p.gn_gamma ? ((e & 1) ? C::hi(gw[e >> 1]) : C::lo(gw[e >> 1])) : 1.0f;
                  const float bet = p.gn_beta ? ((e & 1) ? C::hi(bw[e >> 1]) : C::lo(bw[e >> 1])) : 0.0f;
                  sc[e] = rstd * gam;
                  sh[e] = fmaf(-mean, sc[e], bet);
                }
                const uint32_t base = x_ring + stage * x_stage + pchunk * 16u;
#pragma unroll
                for (int j = 0; j < kRows; ++j) {
                  const int h = rho[j] * p.sh + ih - p.ph;
                  const int w = rwo[j] * p.sw + iw - p.pw;
                  if (h < 0 || h >= p.H || w < 0 || w >= p.W) continue;   // padding (or past the frame)
                  const uint32_t addr = base + (r0 + 16u * j) * 128u;
                  const uint4 q = ld_shared_v4(addr);
                  const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
                  uint32_t o[4];
#pragma unroll
                  for (int e2 = 0; e2 < 4; ++e2) {
                    float a = fmaf(C::lo(qw[e2]), sc[2 * e2], sh[2 * e2]);
                    float b = fmaf(C::hi(qw[e2]), sc[2 * e2 + 1], sh[2 * e2 + 1]);
                    if (p.gn_silu) {
                      a = silu_fast(a);
                      b = silu_fast(b);
                    }
                    o[e2] = C::pack(a, b);
                  }
                  st_shared_v4(addr, o[0], o[1], o[2], o[3]);
                }
              }
              fence_proxy_async_shared();
              __syncwarp();
              if (lane == 0) mbar_arrive(ready_bar + 8 * stage);
              if (++stage == static_cast<uint32_t>(p.stages)) {
                stage = 0;
                phase ^= 1;
              }
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp q drains TMEM lanes [32q, 32q+32) = 32 output pixels of the tile,
    // 32 channels at a time: tcgen05.ld -> + bias + residual (fp32) -> one
    // rounding -> swizzled shared-memory buffer -> TMA store into y viewed as
    // [frames][Ho*Wo][Cout], which clips rows past the frame and channels past
    // Cout.  The residual chunk is fetched by TMA two chunks ahead (the first
    // two before the accumulator is ready).  With 8 epilogue warps two warps
    // share each lane quarter, one taking the even chunks and one the odd.
    using C = Cvt<kBF16>;
    const uint32_t quarter = warp & 3;            // TMEM lanes [32q, 32q+32)
    const uint32_t ew = warp - 2;                 // epilogue warp index, 0..kEpiWarps-1
    const int j0 = kEpi8 ? static_cast<int>(ew) / EPI_WARPS : 0;   // this warp's first chunk
    const uint32_t ybuf = y_stage + ew * kYBufs * ybytes;
    const uint32_t rbuf = r_stage + ew * 2 * EPI_BUF_BYTES;
    const uint32_t rbar = rfull_bar + ew * 16;
    uint32_t rphase[2] = {0, 0};
    bool rpending[2] = {false, false};   // a residual copy into buffer b is in flight
    int local = 0;
    const uint4* bias4 = reinterpret_cast<const uint4*>(p.bias);
    const int chunks = p.BN / 32;
    bool ok = true;
    GnAcc gacc;
    if constexpr (kStats) {
#pragma unroll
      for (int k = 0; k < 8; ++k) gacc.s[k] = gacc.q[k] = 0.0;
      gacc.n = -1;
      gacc.co0 = 0;
    }
    // windows of the accumulator and their offset from the tile's channel base
    const int gn_windows = kSwap ? 1 : p.BN / 32;
    const int gn_off = kSwap ? static_cast<int>(quarter) * 32 : 0;
    if constexpr (kSwap) {
      // Thread = one output channel (TMEM lane), 32 pixels (columns) per chunk.
      for (int i = unit; ok && i < p.num_items; i += num_units, ++local) {
        const uint32_t acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        const Work wk = decode_work<kSplit>(p, i);
        const Tile& tl = wk.tl;
        const bool piece = kSplit && wk.slot >= 0;
        // where this tile's output goes: with mixed output, the fp32 parts of
        // frame 0 through map_f, the other frames 16-bit through map_y
        const bool front_tile = kMixed && tl.to < p.f32_frames;
        const bool f32_tile = p.out_f32 != 0 || front_tile;
        const CUtensorMap* ymap = front_tile ? &map_f : &map_y;
        const int yframe = !kMixed ? tl.frame_out
                           : front_tile      ? tl.n * p.f32_frames + tl.to
                                             : tl.n * p.y_frames + tl.to - p.f32_frames + 1;
        if (kStats && (tl.n != gacc.n || tl.co0 != gacc.co0)) {
          gn_flush(p.gn_out, p.gn_out_groups, p.Cout, gacc, gn_windows, gn_off, lane);
          gacc.n = tl.n;
          gacc.co0 = tl.co0;
        }
        const int ch0 = tl.co0 + static_cast<int>(quarter) * 32;   // this warp's channels
        const bool warp_live = ch0 < p.Cout;
        int live_chunks = (p.HoWo - tl.p0 + 31) / 32;   // pixel chunks inside the frame
        if (live_chunks > chunks) live_chunks = chunks;
        if (!warp_live) live_chunks = 0;
        const int ch = ch0 + static_cast<int>(lane);
        float bv = 0.0f;
        if (p.bias != nullptr && ch < p.Cout)
          bv = C::lo(static_cast<const uint16_t*>(p.bias)[ch]);
        const bool use_res = p.has_residual != 0;
        // the first two residual chunks, fetched ahead of the accumulator (for a
        // tail piece only once it is known to complete the tile)
        auto prefetch_residual = [&]() {
          for (int m = 0; m < 2 && j0 + m * kJStep < live_chunks; ++m) {
            if (lane == 0) {
              mbar_arrive_expect_tx(rbar + 8 * m, EPI_BUF_BYTES);
              tma_load_3d(rbuf + m * EPI_BUF_BYTES, &map_r, rbar + 8 * m, ch0,
                          tl.p0 + 32 * (j0 + m * kJStep), tl.frame_out);
            }
            rpending[m] = true;
          }
        };
        if (use_res && !piece) prefetch_residual();
        bool write_out = true;
        if (!wait_bounded(tfull_bar + 8 * acc, acc_phase, ctl, true)) {
          ok = false;
        } else {
          tc_fence_after();
          const bool has_acc = wk.kb_hi > wk.kb_lo;
          const uint32_t t_row =
              tmem_base + ((quarter * 32u) << 16) + acc * static_cast<uint32_t>(p.BN);
          bool from_parts = false;
          if constexpr (kSplit) {
            if (piece) {
              write_out = store_piece(p, wk.slot, t_row, has_acc, quarter, lane, j0, kJStep, ew);
              from_parts = write_out;
              if (write_out && use_res) prefetch_residual();
            }
          }
          // byte offset of (pixel e, this thread's channel) in a 32 x 32 buffer
          const uint32_t col_byte = (lane & 7u) * 2u;
          for (int j = j0, m = 0; write_out && j < live_chunks; j += kJStep, ++m) {
            const uint32_t b = m & 1;
            float v[32];
            if (kSplit && from_parts) {
              sum_pieces(p, wk.slot - wk.slot % p.split_s, quarter * 32u + lane, j, v);
            } else {
              uint32_t r[32];
              tmem_ld_32x32b_x32(t_row + j * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = has_acc ? __uint_as_float(r[e]) : 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] += bv;
            if (use_res) {
              if (!wait_bounded(rbar + 8 * b, rphase[b], ctl, true)) {
                ok = false;
                break;
              }
              rphase[b] ^= 1;
              rpending[b] = false;
              const uint32_t rb = rbuf + b * EPI_BUF_BYTES;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                uint16_t q;
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(q)
                             : "r"(rb + swz64(e, lane >> 3) + col_byte)
                             : "memory");
                v[e] += C::lo(q);
              }
            }
            if (lane == 0) bulk_wait_group_read<kYBufs - 1>();
            __syncwarp();
            const uint32_t yb = ybuf + (m & (kYBufs - 1)) * ybytes;
            if (f32_tile) {
              // fp32 rows of 32 channels (128 bytes, 128-byte swizzle): this
              // thread's channel is 4-byte word (lane & 3) of 16-byte chunk lane >> 2
              const uint32_t word = (lane & 3u) * 4u;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(yb + swz128(e, lane >> 2) + word),
                             "f"(v[e])
                             : "memory");
            } else if (kScatter) {
              // strided output: lane = channel, so each pixel's 32 channels are
              // one 64-byte store of the warp
              int q = tl.p0 + 32 * j;
              int a = q / p.Wo, bq = q - a * p.Wo;
#pragma unroll 4
              for (int e = 0; e < 32; ++e, ++q) {
                if (q < p.HoWo && ch < p.Cout) {
                  const size_t off =
                      ((static_cast<size_t>(yframe) * p.sc_H + a * p.sc_sh + p.sc_rh) *
                           p.sc_W + bq * p.sc_sw + p.sc_rw) * p.Cout + ch;
                  p.y_scatter[off] = static_cast<uint16_t>(C::pack(v[e], 0.0f) & 0xFFFFu);
                }
                if (++bq == p.Wo) {
                  bq = 0;
                  ++a;
                }
              }
            } else {
              float gs = 0.0f, gq = 0.0f;   // this channel's rounded outputs, for the statistics
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const uint16_t q = static_cast<uint16_t>(C::pack(v[e], 0.0f) & 0xFFFFu);
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(yb + swz64(e, lane >> 3) + col_byte),
                             "h"(q)
                             : "memory");
                if (kStats && tl.p0 + 32 * j + e < p.HoWo) {
                  const float yv = C::lo(q);
                  gs += yv;
                  gq = fmaf(yv, yv, gq);
                }
              }
              if constexpr (kStats) {
                // lane = channel ch: its pixels' sums go to its own accumulator
                gacc.s[0] += gs;
                gacc.q[0] += gq;
              }
            }
            fence_proxy_async_shared();
            __syncwarp();
            const int pix0 = tl.p0 + 32 * j;
            const bool refill = use_res && j + 2 * kJStep < live_chunks;
            if (lane == 0) {
              if (!kScatter || f32_tile) {   // strided 16-bit frames were stored above
                tma_store_3d(ymap, yb, ch0, pix0, yframe);
                bulk_commit_group();
              }
              if (refill) {
                mbar_arrive_expect_tx(rbar + 8 * b, EPI_BUF_BYTES);
                tma_load_3d(rbuf + b * EPI_BUF_BYTES, &map_r, rbar + 8 * b, ch0,
                            pix0 + 64 * kJStep, tl.frame_out);
              }
            }
            if (refill) rpending[b] = true;
          }
        }
        if (!ok && lane == 0) {
          for (int j = 0; j < 2; ++j)
            if (rpending[j]) wait_bounded(rbar + 8 * j, rphase[j], ctl, false);
        }
        if (!ok) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar + 8 * acc);
      }
    } else
    for (int i = unit; ok && i < p.num_items; i += num_units, ++local) {
      const uint32_t acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const Work wk = decode_work<kSplit>(p, i);
      const Tile& tl = wk.tl;
      const bool piece = kSplit && wk.slot >= 0;
      // where this tile's output goes: with mixed output, the fp32 parts of
      // frame 0 through map_f, the other frames 16-bit through map_y
      const bool front_tile = kMixed && tl.to < p.f32_frames;
      const bool f32_tile = p.out_f32 != 0 || front_tile;
      const CUtensorMap* ymap = front_tile ? &map_f : &map_y;
      const int yframe = !kMixed ? tl.frame_out
                         : front_tile      ? tl.n * p.f32_frames + tl.to
                                           : tl.n * p.y_frames + tl.to - p.f32_frames + 1;
      if (kStats && (tl.n != gacc.n || tl.co0 != gacc.co0)) {
        gn_flush(p.gn_out, p.gn_out_groups, p.Cout, gacc, gn_windows, gn_off, lane);
        gacc.n = tl.n;
        gacc.co0 = tl.co0;
      }
      const int row_base = tl.p0 + static_cast<int>(rank) * BM + static_cast<int>(quarter) * 32;
      const bool rows_live = row_base < p.HoWo;   // some of this warp's rows are in the frame
      // channel chunks that hold at least one real output channel
      int live_chunks = (p.Cout - tl.co0 + 31) / 32;
      if (live_chunks > chunks) live_chunks = chunks;
      const bool use_res = p.has_residual && rows_live;
      // the first two residual chunks, fetched ahead of the accumulator (for a
      // tail piece only once it is known to complete the tile)
      auto prefetch_residual = [&]() {
        for (int m = 0; m < 2 && j0 + m * kJStep < live_chunks; ++m) {
          if (lane == 0) {
            mbar_arrive_expect_tx(rbar + 8 * m, EPI_BUF_BYTES);
            tma_load_3d(rbuf + m * EPI_BUF_BYTES, &map_r, rbar + 8 * m,
                        tl.co0 + 32 * (j0 + m * kJStep), row_base, tl.frame_out);
          }
          rpending[m] = true;
        }
      };
      if (use_res && !piece) prefetch_residual();
      bool write_out = true;
      if (!wait_bounded(tfull_bar + 8 * acc, acc_phase, ctl, true)) {
        ok = false;
      } else {
        tc_fence_after();
        const bool has_acc = wk.kb_hi > wk.kb_lo;
        const uint32_t t_row =
            tmem_base + ((quarter * 32u) << 16) + acc * static_cast<uint32_t>(p.BN);
        bool from_parts = false;
        if constexpr (kSplit) {
          if (piece) {
            write_out = store_piece(p, wk.slot, t_row, has_acc, quarter, lane, j0, kJStep, ew);
            from_parts = write_out;
            if (write_out && use_res) prefetch_residual();
          }
        }
        for (int j = j0, m = 0; write_out && rows_live && j < live_chunks; j += kJStep, ++m) {
          const uint32_t b = m & 1;
          float v[32];
          if (kSplit && from_parts) {
            sum_pieces(p, wk.slot - wk.slot % p.split_s, quarter * 32u + lane, j, v);
          } else {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + j * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = has_acc ? __uint_as_float(r[e]) : 0.0f;
          }
          const int cb = tl.co0 + j * 32;
          if (bias4 != nullptr) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (cb + 8 * g < p.Cout) {
                const uint4 q = __ldg(bias4 + cb / 8 + g);
                v[8 * g + 0] += C::lo(q.x); v[8 * g + 1] += C::hi(q.x);
                v[8 * g + 2] += C::lo(q.y); v[8 * g + 3] += C::hi(q.y);
                v[8 * g + 4] += C::lo(q.z); v[8 * g + 5] += C::hi(q.z);
                v[8 * g + 6] += C::lo(q.w); v[8 * g + 7] += C::hi(q.w);
              }
            }
          }
          if (use_res) {
            if (!wait_bounded(rbar + 8 * b, rphase[b], ctl, true)) {
              ok = false;
              break;
            }
            rphase[b] ^= 1;
            rpending[b] = false;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const uint4 q = ld_shared_v4(rbuf + b * EPI_BUF_BYTES + swz64(lane, g));
              v[8 * g + 0] += C::lo(q.x); v[8 * g + 1] += C::hi(q.x);
              v[8 * g + 2] += C::lo(q.y); v[8 * g + 3] += C::hi(q.y);
              v[8 * g + 4] += C::lo(q.z); v[8 * g + 5] += C::hi(q.z);
              v[8 * g + 6] += C::lo(q.w); v[8 * g + 7] += C::hi(q.w);
            }
          }
          // the store issued from this buffer two chunks ago must have read it
          if (lane == 0) bulk_wait_group_read<kYBufs - 1>();
          __syncwarp();
          const uint32_t yb = ybuf + (m & (kYBufs - 1)) * ybytes;
          if (f32_tile) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              st_shared_v4(yb + swz128(lane, c), __float_as_uint(v[4 * c + 0]),
                           __float_as_uint(v[4 * c + 1]), __float_as_uint(v[4 * c + 2]),
                           __float_as_uint(v[4 * c + 3]));
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int g = 0; g < 16; ++g) pk[g] = C::pack(v[2 * g], v[2 * g + 1]);
            if constexpr (kScatter) {
              // strided output: this thread's pixel, 32 channels as four 16-byte stores
              const int q = row_base + static_cast<int>(lane);
              if (q < p.HoWo) {
                const int a = q / p.Wo, bq = q - a * p.Wo;
                uint4* dst = reinterpret_cast<uint4*>(
                    p.y_scatter +
                    ((static_cast<size_t>(yframe) * p.sc_H + a * p.sc_sh + p.sc_rh) *
                         p.sc_W + bq * p.sc_sw + p.sc_rw) * p.Cout + cb);
#pragma unroll
                for (int g = 0; g < 4; ++g)
                  if (cb + 8 * g < p.Cout)
                    dst[g] = make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
              }
            } else {
#pragma unroll
              for (int g = 0; g < 4; ++g)
                st_shared_v4(yb + swz64(lane, g), pk[4 * g], pk[4 * g + 1],
                             pk[4 * g + 2], pk[4 * g + 3]);
            }
            if constexpr (kStats) {
              // lane = channel cb + lane: its column of the staged 32 x 32
              // block (the rows inside the frame), read back from shared memory
              __syncwarp();
              int rows_in = p.HoWo - row_base;
              if (rows_in > 32) rows_in = 32;
              const uint32_t col = yb + (lane & 7u) * 2u;
              float gs = 0.0f, gq = 0.0f;
              for (int e = 0; e < rows_in; ++e) {
                uint16_t qv;
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(qv)
                             : "r"(col + swz64(static_cast<uint32_t>(e), lane >> 3))
                             : "memory");
                const float yv = C::lo(qv);
                gs += yv;
                gq = fmaf(yv, yv, gq);
              }
              gacc.s[j] += gs;
              gacc.q[j] += gq;
            }
          }
          fence_proxy_async_shared();
          __syncwarp();
          // every lane has read residual buffer b: refill it with chunk j+2
          const bool refill = use_res && j + 2 * kJStep < live_chunks;
          if (lane == 0) {
            if (!kScatter || f32_tile) {   // strided 16-bit frames were stored above
              tma_store_3d(ymap, yb, cb, row_base, yframe);
              bulk_commit_group();
            }
            if (refill) {
              mbar_arrive_expect_tx(rbar + 8 * b, EPI_BUF_BYTES);
              tma_load_3d(rbuf + b * EPI_BUF_BYTES, &map_r, rbar + 8 * b, cb + 64 * kJStep,
                          row_base, tl.frame_out);
            }
          }
          if (refill) rpending[b] = true;
        }
      }
      if (!ok && lane == 0) {
        // residual copies of this tile still in flight must land before exit
        for (int j = 0; j < 2; ++j)
          if (rpending[j]) wait_bounded(rbar + 8 * j, rphase[j], ctl, false);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair)
          mbar_arrive_cluster(mapa_shared(tempty_bar + 8 * acc, 0));
        else
          mbar_arrive(tempty_bar + 8 * acc);
      }
    }
    if constexpr (kStats) gn_flush(p.gn_out, p.gn_out_groups, p.Cout, gacc, gn_windows, gn_off, lane);
    // y stores must be complete (and their shared-memory sources read) before exit
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();   // no CTA leaves while its peer may touch it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else
      tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// First-frame fold (Qwen Image post, "Video VAE": when the frames before the
// first are padding, the 3D conv of a single frame is a 2D conv with adjusted
// weights; with replicate padding every temporal tap reads frame 0, so the
// adjusted 2D weight is the sum over the temporal taps).  The sum s is taken
// in fp32 and stored as two 16-bit parts, hi = round(s) and
// lo = round(s - hi), laid out as a kt = 2 weight [Cout][2][kh*kw*Cin]:
// both parts multiply the same frame, so the folded conv carries about 16
// significant bits of the adjusted weight instead of 8 (a single rounding of
// s alone adds an error comparable to the output rounding).
template <bool kBF16>
__global__ void fold_temporal_taps_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ w2,
                                          int Cout, int kt, int spatial_cin) {
  using C = Cvt<kBF16>;
  // the convolution that reads w2 waits for this whole grid before reading
  griddep_launch_dependents();
  // thread = 8 consecutive entries (16 bytes) of one output channel's row:
  // spatial_cin is a multiple of 8 and both weights are 16-byte aligned
  const int vecs = spatial_cin / 8;
  const long long total = static_cast<long long>(Cout) * vecs;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long co = i / vecs;
    const long long rest = (i - co * vecs) * 8;
    float s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int it = 0; it < kt; ++it) {
      const uint4 v = *reinterpret_cast<const uint4*>(w + (co * kt + it) * spatial_cin + rest);
      s[0] += C::lo(v.x); s[1] += C::hi(v.x); s[2] += C::lo(v.y); s[3] += C::hi(v.y);
      s[4] += C::lo(v.z); s[5] += C::hi(v.z); s[6] += C::lo(v.w); s[7] += C::hi(v.w);
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hi[q] = C::pack(s[2 * q], s[2 * q + 1]);
      lo[q] = C::pack(s[2 * q] - C::lo(hi[q]), s[2 * q + 1] - C::hi(hi[q]));
    }
    *reinterpret_cast<uint4*>(w2 + co * 2 * spatial_cin + rest) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(w2 + co * 2 * spatial_cin + spatial_cin + rest) =
        make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// The same fold with the lo part in 8 bits: hi = round16(s) into w2
// ([Cout][kh*kw*Cin], 16-bit) and lo8 = e5m2((s - hi) * 2^8) into w8 (same
// layout, one byte each).  The x operand of the lo product is e5m2(x * 2^-8)
// (x_to_e5m2_kernel), so the scales cancel in the product.  e5m2 keeps 3
// significant bits: the lo product's error is about 2^-3 of a term that is
// itself at most 2^-8 of the weight, below the output's 16-bit rounding; the
// scales keep both operands in e5m2's normal range (2^-14 .. 57344) for
// weights above 2^-14 and activations up to 1.4e7.
template <bool kBF16>
__global__ void fold_taps_lo8_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ w2,
                                     uint8_t* __restrict__ w8, int Cout, int kt, int spatial_cin) {
  using C = Cvt<kBF16>;
  griddep_launch_dependents();
  const int vecs = spatial_cin / 8;
  const long long total = static_cast<long long>(Cout) * vecs;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long co = i / vecs;
    const long long rest = (i - co * vecs) * 8;
    float s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int it = 0; it < kt; ++it) {
      const uint4 v = *reinterpret_cast<const uint4*>(w + (co * kt + it) * spatial_cin + rest);
      s[0] += C::lo(v.x); s[1] += C::hi(v.x); s[2] += C::lo(v.y); s[3] += C::hi(v.y);
      s[4] += C::lo(v.z); s[5] += C::hi(v.z); s[6] += C::lo(v.w); s[7] += C::hi(v.w);
    }
    uint32_t hi[4], lo[2];
#pragma unroll
    for (int q = 0; q < 4; ++q) hi[q] = C::pack(s[2 * q], s[2 * q + 1]);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t a = e5m2x2(256.0f * (s[4 * q] - C::lo(hi[2 * q])),
                                256.0f * (s[4 * q + 1] - C::hi(hi[2 * q])));
      const uint32_t b = e5m2x2(256.0f * (s[4 * q + 2] - C::lo(hi[2 * q + 1])),
                                256.0f * (s[4 * q + 3] - C::hi(hi[2 * q + 1])));
      lo[q] = a | (b << 16);
    }
    *reinterpret_cast<uint4*>(w2 + co * spatial_cin + rest) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint2*>(w8 + co * spatial_cin + rest) = make_uint2(lo[0], lo[1]);
  }
}

// x8 = e5m2(x * 2^-8), 8 values per thread (n a multiple of 8).
template <bool kBF16>
__global__ void x_to_e5m2_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ x8,
                                 long long n) {
  using C = Cvt<kBF16>;
  // the convolution that reads x8 waits for this whole grid before reading
  griddep_launch_dependents();
  const float sc = 1.0f / 256.0f;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n / 8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t a = e5m2x2(sc * C::lo(v.x), sc * C::hi(v.x)) | (e5m2x2(sc * C::lo(v.y), sc * C::hi(v.y)) << 16);
    const uint32_t b = e5m2x2(sc * C::lo(v.z), sc * C::hi(v.z)) | (e5m2x2(sc * C::lo(v.w), sc * C::hi(v.w)) << 16);
    reinterpret_cast<uint2*>(x8)[i] = make_uint2(a, b);
  }
}

// Backward data pass: the weight the transposed convolution runs with,
// wt[ci, it, ih, iw, co] = w[co, kt-1-it, kh-1-ih, kw-1-iw, ci] (every tap
// mirrored, the channel roles exchanged).  Mirroring all three tap indices
// reverses the linear tap order, so each tap is a [Cout x Cin] -> [Cin x Cout]
// transpose: block = one tap and a 64 x 64 tile, staged in shared memory so
// that both the reads and the writes run along contiguous channels.
// Launch: grid (ceil(Cin/64), ceil(Cout/64), taps), block (32, 8).
//
// With a spatial stride the data gradient splits into phases (rh, rw): dx rows
// a*sh + rh receive only the taps ih = qh + sh*j (qh = (rh + ph) mod sh), so a
// phase is a convolution of dy with the sub-kernel of those taps, mirrored.
// Then wt holds that sub-kernel: wt[ci, it', jh', jw', co] =
// w[co, kt-1-it', qh + sh*(Jh-1-jh'), qw + sw*(Jw-1-jw'), ci], taps = kt*Jh*Jw
// (sh = sw = 1, qh = qw = 0, Jh = kh, Jw = kw: the plain mirror above).
__global__ void flip_transpose_weight_kernel(const uint16_t* __restrict__ w,
                                             uint16_t* __restrict__ wt, int Cout, int taps,
                                             int Cin, int kh, int kw, int Jh, int Jw, int qh,
                                             int qw, int sh, int sw) {
  // 64 x 64 tile, two 16-bit values (4 bytes) per thread access: Cin and Cout
  // are even, so a pair never straddles the end of a row
  __shared__ __align__(4) uint16_t tile[64][66];    // [co][ci], 33-word rows
  const int ci0 = blockIdx.x * 64, co0 = blockIdx.y * 64;
  const int tap = blockIdx.z;                  // tap of wt: (it', jh', jw')
  const int jw_ = tap % Jw, jh_ = (tap / Jw) % Jh, it_ = tap / (Jw * Jh);
  const int kt = taps / (Jh * Jw);
  const int tap_src = ((kt - 1 - it_) * kh + qh + sh * (Jh - 1 - jh_)) * kw + qw + sw * (Jw - 1 - jw_);
  const int taps_src = kt * kh * kw;
  const int x2 = 2 * static_cast<int>(threadIdx.x);
  for (int r = threadIdx.y; r < 64; r += 8) {
    const int co = co0 + r, ci = ci0 + x2;
    if (co < Cout && ci < Cin)
      *reinterpret_cast<uint32_t*>(&tile[r][x2]) = *reinterpret_cast<const uint32_t*>(
          w + (static_cast<long long>(co) * taps_src + tap_src) * Cin + ci);
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 64; r += 8) {
    const int ci = ci0 + r, co = co0 + x2;
    if (co < Cout && ci < Cin)
      *reinterpret_cast<uint32_t*>(wt + (static_cast<long long>(ci) * taps + tap) * Cout + co) =
          static_cast<uint32_t>(tile[x2][r]) | (static_cast<uint32_t>(tile[x2 + 1][r]) << 16);
  }
}

// The single-frame data gradient's weight in one pass: the transposed
// convolution's weight (every tap mirrored, Cin and Cout exchanged) with its kt
// temporal taps summed and split into hi and lo 16-bit parts, as the first-frame
// fold does -- w2[ci][0][jh][jw][co] = hi(s), w2[ci][1][jh][jw][co] = lo(s) with
// s = sum over it of w[co][it][kh-1-jh][kw-1-jw][ci], summed in fp32.  Block =
// one spatial tap and a 64 x 64 (co, ci) tile; the sums are staged in shared
// memory so that reads and writes both run along contiguous channels.
// Launch: grid (ceil(Cin/64), ceil(Cout/64), kh*kw), block (32, 8).
template <bool kBF16>
__global__ void flip_fold_weight_kernel(const uint16_t* __restrict__ w,
                                        uint16_t* __restrict__ w2, int Cout, int kt, int kh,
                                        int kw, int Cin) {
  using C = Cvt<kBF16>;
  griddep_launch_dependents();
  __shared__ float tile[64][65];                  // [co][ci] sums
  const int ci0 = blockIdx.x * 64, co0 = blockIdx.y * 64;
  const int tap = blockIdx.z;                     // (jh, jw) of w2
  const int taps2 = kh * kw;
  const int src_sp = taps2 - 1 - tap;             // mirrored spatial tap of w
  const int x2 = 2 * static_cast<int>(threadIdx.x);
  // rows ty, ty + 8, ..., ty + 56: eight loads in flight per temporal tap
  float a[8], b[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = b[k] = 0.0f;
  const int ci = ci0 + x2;
  for (int it = 0; it < kt; ++it) {
    uint32_t v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int co = co0 + static_cast<int>(threadIdx.y) + 8 * k;
      v[k] = (co < Cout && ci < Cin)
                 ? *reinterpret_cast<const uint32_t*>(
                       w + ((static_cast<long long>(co) * kt + it) * taps2 + src_sp) * Cin + ci)
                 : 0u;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      a[k] += C::lo(v[k]);
      b[k] += C::hi(v[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    tile[threadIdx.y + 8 * k][x2] = a[k];
    tile[threadIdx.y + 8 * k][x2 + 1] = b[k];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 64; r += 8) {
    const int ci = ci0 + r, co = co0 + x2;
    if (co < Cout && ci < Cin) {
      const float a = tile[x2][r], b = tile[x2 + 1][r];
      const uint32_t hi = C::pack(a, b);
      const uint32_t lo = C::pack(a - C::lo(hi), b - C::hi(hi));
      const long long row = static_cast<long long>(ci) * 2 * taps2;
      *reinterpret_cast<uint32_t*>(w2 + (row + tap) * Cout + co) = hi;
      *reinterpret_cast<uint32_t*>(w2 + (row + taps2 + tap) * Cout + co) = lo;
    }
  }
}

// Causal replicate padding reads frame 0 for the kt-1 frames in front, so the
// gradient of those virtual frames belongs to frame 0: dx[n, 0] = sum of
// ext[n, 0 .. kt-1], ext holding the fp32 gradient of the kt frames
// -(kt-1)..0 (frame 0's own taps in ext[n, kt-1]); one rounding.  Frames >= 1
// are written by the convolution itself.  8 values per thread.
//
// Strided phases: ext holds a phase's A_h x A_w pixels per frame, and pixel
// (a, b) of it belongs at row a*sh + rh, column b*sw + rw of dx's H x W frame
// (phase = nullptr: ext's frames are dx's, pixel for pixel).
struct FoldPhase {
  int Aw, sh, sw, rh, rw, H, W, C;
};

template <bool kBF16>
__global__ void fold_front_gradient_kernel(const float* __restrict__ ext,
                                           uint16_t* __restrict__ dx, int N, int D, int kt,
                                           long long frame_elems, FoldPhase ph, int phased) {
  using C = Cvt<kBF16>;
  const long long vecs_per_frame = frame_elems / 8;
  const long long total = static_cast<long long>(N) * vecs_per_frame;
  const float4* e4 = reinterpret_cast<const float4*>(ext);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long v = i % vecs_per_frame;
    const long long n = i / vecs_per_frame;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int e = 0; e < kt; ++e) {
      const long long at = ((n * kt + e) * vecs_per_frame + v) * 2;
      const float4 a = e4[at], b = e4[at + 1];
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    uint4 out;
    out.x = C::pack(acc[0], acc[1]);
    out.y = C::pack(acc[2], acc[3]);
    out.z = C::pack(acc[4], acc[5]);
    out.w = C::pack(acc[6], acc[7]);
    if (!phased) {
      reinterpret_cast<uint4*>(dx)[n * D * vecs_per_frame + v] = out;
    } else {
      const long long pix = (v * 8) / ph.C, c = (v * 8) - pix * ph.C;
      const long long a = pix / ph.Aw, b = pix - a * ph.Aw;
      const long long off =
          ((n * D * static_cast<long long>(ph.H) + a * ph.sh + ph.rh) * ph.W + b * ph.sw + ph.rw) *
              ph.C + c;
      *reinterpret_cast<uint4*>(dx + off) = out;
    }
  }
}

// dx positions of a phase that no tap reaches (a stride larger than the
// kernel): every frame's rows a*sh + rh, columns b*sw + rw, all channels,
// set to zero.  8 channels (16 bytes) per thread.
__global__ void zero_phase_kernel(uint16_t* __restrict__ dx, long long frames, int Ah, int Aw,
                                  FoldPhase ph) {
  const long long vecs_per_pix = ph.C / 8;
  const long long total = frames * Ah * Aw * vecs_per_pix;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = (i % vecs_per_pix) * 8;
    long long pix = i / vecs_per_pix;
    const long long b = pix % Aw;
    pix /= Aw;
    const long long a = pix % Ah;
    const long long f = pix / Ah;
    const long long off = ((f * ph.H + a * ph.sh + ph.rh) * ph.W + b * ph.sw + ph.rw) * ph.C + c;
    *reinterpret_cast<uint4*>(dx + off) = make_uint4(0, 0, 0, 0);
  }
}

}  // namespace conv3d
