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
// One CTA per SM, persistent over output tiles of BM = 128 pixels x BN output
// channels.  Warp roles (192 threads):
//   warp 0     TMA producer: per k-block one im2col load of A (128 pixels x 64
//              channels of one tap) and one tiled load of B (BN x 64), both
//              128-byte swizzled, into a ring of `stages` shared-memory slots
//              guarded by full/empty mbarriers;
//   warp 1     allocates tensor memory and issues tcgen05.mma (M=128, N=BN,
//              K=16, four per k-block) into one of two fp32 TMEM accumulators;
//   warps 2-5  epilogue: tcgen05.ld, + bias, + residual, one rounding to the
//              output type, 16-byte stores; then frees the accumulator so the
//              next tile's main loop overlaps this tile's epilogue.
// Every mbarrier wait is bounded in time; a wait that runs out records
// CONV3D_ERR_TIMEOUT in the status word, and all roles leave their loops,
// drain their asynchronous work and free tensor memory before exiting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace conv3d {

constexpr int BM = 128;             // output pixels per tile (TMEM lanes)
constexpr int BK = 64;              // channels per k-block (128 bytes of fp16/bf16)
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr int MAX_STAGES = 8;

constexpr int STATUS_TIMEOUT = 5;   // mirrors CONV3D_ERR_TIMEOUT

struct KernelParams {
  int D, Do, Ho, Wo;                 // input frames; output extents
  int HoWo;
  int Cin, Cout;
  int kt, kh, kw;
  int pf, ph, pw;                    // front temporal pad, spatial pads
  int tpad;                          // 0 zero, 1 causal replicate, 2 causal zero
  int n_chunks;                      // ceil(Cin / BK)
  int BN;                            // output channels per tile (multiple of 32, <= 256)
  int n_tiles_n;                     // ceil(Cout / BN)
  int tiles_per_frame;               // ceil(HoWo / BM)
  int num_tiles;
  int stages;
  uint32_t tmem_cols;                // power of two >= 2*BN
  uint32_t idesc;
  const void* bias;                  // [Cout] or null
  const void* residual;              // [M, Cout] or null
  void* y;                           // [M, Cout]
  int* status;                       // device status word
  unsigned long long timeout_ns;
};

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
  r.p0 = (mt - r.frame_out * p.tiles_per_frame) * BM;
  r.n = r.frame_out / p.Do;
  r.to = r.frame_out - r.n * p.Do;
  r.co0 = nt * p.BN;
  return r;
}

// Source frame read by temporal tap `it` of output frame `to`, or -1 when the
// tap reads zero padding (and contributes nothing).
__device__ __forceinline__ int source_frame(const KernelParams& p, int to, int it) {
  int f = to + it - p.pf;
  if (f < 0) return p.tpad == 1 ? 0 : -1;
  return f < p.D ? f : -1;
}

__device__ __forceinline__ int kblocks_of_tile(const KernelParams& p, int to) {
  int valid = 0;
  for (int it = 0; it < p.kt; ++it) valid += source_frame(p, to, it) >= 0;
  return valid * p.kh * p.kw * p.n_chunks;
}

struct SharedCtl {
  volatile int* abort_flag;
  int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void raise_abort(const SharedCtl& c, int code) {
  *c.abort_flag = 1;
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

template <bool kBF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    conv3d_implicit_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                const __grid_constant__ CUtensorMap map_b,
                                const KernelParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;

  const uint32_t warp = threadIdx.x / 32;
  const uint32_t lane = threadIdx.x % 32;

  // Carve shared memory: A ring, B ring (both 1024-byte aligned for the
  // 128-byte swizzle), then the mbarriers.
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t b_stage_bytes = static_cast<uint32_t>(p.BN) * BK * 2;
  const uint32_t a_ring = base;
  const uint32_t b_ring = a_ring + p.stages * A_STAGE_BYTES;
  const uint32_t bars = b_ring + p.stages * b_stage_bytes;
  const uint32_t full_bar = bars;                         // [stages]
  const uint32_t empty_bar = bars + 8 * p.stages;         // [stages]
  const uint32_t tfull_bar = bars + 16 * p.stages;        // [2]
  const uint32_t tempty_bar = tfull_bar + 16;             // [2]
  const uint32_t drain_bar = tempty_bar + 16;             // [1]

  SharedCtl ctl{&s_abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar + 8 * a, 1);
      mbar_init(tempty_bar + 8 * a, 4);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&s_tmem_base), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t tx_bytes = A_STAGE_BYTES + b_stage_bytes;
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        const Tile tl = decode_tile(p, t);
        const int ho0 = tl.p0 / p.Wo;
        const int wo0 = tl.p0 - ho0 * p.Wo;
        const int w_org = wo0 - p.pw;   // window origin of the tile's first pixel
        const int h_org = ho0 - p.ph;
        for (int it = 0; ok && it < p.kt; ++it) {
          const int f = source_frame(p, tl.to, it);
          if (f < 0) continue;
          const int img = tl.n * p.D + f;
          for (int ih = 0; ok && ih < p.kh; ++ih) {
            for (int iw = 0; ok && iw < p.kw; ++iw) {
              const int tap = (it * p.kh + ih) * p.kw + iw;
              for (int cc = 0; cc < p.n_chunks; ++cc) {
                if (!wait_bounded(empty_bar + 8 * stage, phase ^ 1, ctl, true)) {
                  ok = false;
                  break;
                }
                mbar_arrive_expect_tx(full_bar + 8 * stage, tx_bytes);
                tma_load_im2col_4d(a_ring + stage * A_STAGE_BYTES, &map_a, full_bar + 8 * stage,
                                   cc * BK, w_org, h_org, img, static_cast<uint16_t>(iw),
                                   static_cast<uint16_t>(ih));
                tma_load_3d(b_ring + stage * b_stage_bytes, &map_b, full_bar + 8 * stage,
                            cc * BK, tap, tl.co0);
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
      if (!ok) {
        // Let the copies already in flight land before the CTA may exit.
        const long long first = issued > p.stages ? issued - p.stages : 0;
        for (long long i = first; i < issued; ++i) {
          const uint32_t s = static_cast<uint32_t>(i % p.stages);
          const uint32_t par = static_cast<uint32_t>((i / p.stages) & 1);
          wait_bounded(full_bar + 8 * s, par, ctl, false);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int local = 0;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++local) {
        const Tile tl = decode_tile(p, t);
        const int nkb = kblocks_of_tile(p, tl.to);
        const uint32_t acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!wait_bounded(tempty_bar + 8 * acc, acc_phase ^ 1, ctl, true)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(p.BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_bounded(full_bar + 8 * stage, phase, ctl, true)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc_k_sw128(a_ring + stage * A_STAGE_BYTES);
          const uint64_t db = smem_desc_k_sw128(b_ring + stage * b_stage_bytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // +32 bytes along K inside the swizzled 128-byte row = +2 in the
            // descriptor's address field.
            mma_f16_ss(d_tmem, da + 2 * k, db + 2 * k, p.idesc, (kb | k) != 0);
          }
          mma_commit(empty_bar + 8 * stage);
          if (++stage == static_cast<uint32_t>(p.stages)) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(tfull_bar + 8 * acc);
      }
      // All tensor-core work of this CTA has finished once the drain fires.
      mma_commit(drain_bar);
      wait_bounded(drain_bar, 0, ctl, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    using C = Cvt<kBF16>;
    const uint32_t quarter = warp & 3;            // TMEM lanes [32q, 32q+32)
    const int row = static_cast<int>(quarter * 32 + lane);
    int local = 0;
    const uint4* bias4 = reinterpret_cast<const uint4*>(p.bias);
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++local) {
      const uint32_t acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!wait_bounded(tfull_bar + 8 * acc, acc_phase, ctl, true)) break;
      tc_fence_after();
      const Tile tl = decode_tile(p, t);
      const bool has_acc = kblocks_of_tile(p, tl.to) > 0;
      const int pix = tl.p0 + row;
      const bool row_ok = pix < p.HoWo;
      const long long m = static_cast<long long>(tl.frame_out) * p.HoWo + pix;
      const uint32_t t_row = tmem_base + ((quarter * 32u) << 16) + acc * static_cast<uint32_t>(p.BN);
      for (int j = 0; j < p.BN / 32; ++j) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + j * 32, r);
        tmem_ld_wait();
        const int cb = tl.co0 + j * 32;
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int co = cb + g * 8;
            if (co < p.Cout) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = has_acc ? __uint_as_float(r[g * 8 + e]) : 0.0f;
              if (bias4 != nullptr) {
                const uint4 b = __ldg(bias4 + co / 8);
                v[0] += C::lo(b.x); v[1] += C::hi(b.x); v[2] += C::lo(b.y); v[3] += C::hi(b.y);
                v[4] += C::lo(b.z); v[5] += C::hi(b.z); v[6] += C::lo(b.w); v[7] += C::hi(b.w);
              }
              const long long off = m * p.Cout + co;  // element offset, multiple of 8
              if (p.residual != nullptr) {
                const uint4 q = *reinterpret_cast<const uint4*>(
                    static_cast<const uint16_t*>(p.residual) + off);
                v[0] += C::lo(q.x); v[1] += C::hi(q.x); v[2] += C::lo(q.y); v[3] += C::hi(q.y);
                v[4] += C::lo(q.z); v[5] += C::hi(q.z); v[6] += C::lo(q.w); v[7] += C::hi(q.w);
              }
              uint4 o;
              o.x = C::pack(v[0], v[1]);
              o.y = C::pack(v[2], v[3]);
              o.z = C::pack(v[4], v[5]);
              o.w = C::pack(v[6], v[7]);
              *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + off) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar + 8 * acc);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
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
  const long long total = static_cast<long long>(Cout) * spatial_cin;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long co = i / spatial_cin;
    const long long rest = i - co * spatial_cin;
    float s = 0.0f;
    for (int it = 0; it < kt; ++it) {
      const uint32_t v = w[(co * kt + it) * spatial_cin + rest];
      s += C::lo(v);
    }
    const uint32_t hi = C::pack(s, 0.0f) & 0xFFFFu;
    const uint32_t lo = C::pack(s - C::lo(hi), 0.0f) & 0xFFFFu;
    w2[co * 2 * spatial_cin + rest] = static_cast<uint16_t>(hi);
    w2[co * 2 * spatial_cin + spatial_cin + rest] = static_cast<uint16_t>(lo);
  }
}

}  // namespace conv3d
