// groupnorm.cu -- GroupNorm statistics and the fused normalise + SiLU pass
// that precede each decoder convolution (stable-diffusion.cpp discussion
// "Exe Heavy Metal": GROUP_NORM on the GPU; news.bugfactory.tech: a fused
// GroupNorm + SiLU kernel).  Both passes are HBM-bound and touch each element
// once (statistics: one read; apply: one read and one write), so they run as
// two plain streaming kernels with 16-byte vector accesses rather than inside
// the convolution, whose im2col operand would repeat the transform once per
// filter tap.
//
// Layout: x and y are [N, D, H, W, C] (NDHWC).  A statistic set is one sample
// (all D*H*W pixels) or, with per_frame, one frame of one sample (H*W pixels).
// stats is [sets][groups][2] fp64.  The statistics pass accumulates {sum of
// x, sum of x^2} over the set's pixels and the group's C/groups channels and
// then turns each pair into {mean, 1/sqrt(var + eps)} in place (biased
// variance), which is what the apply pass reads.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "conv3d.h"

// Defined beside the convolution kernels: counts `n` launches just enqueued
// (conv3d_kernel_launches) and returns their status.
cudaError_t conv3d_count_launches(int n);

namespace conv3d_gn {

template <bool kBF16>
__device__ __forceinline__ float to_f(uint32_t bits16) {
  if (kBF16) return __uint_as_float(bits16 << 16);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)));
}

// Two values rounded (nearest even) into one 32-bit pair, the first in the low half.
template <bool kBF16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if (kBF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// SiLU with one special-function operation: silu(z) = z * sigmoid(z) and
// sigmoid(z) = (1 + tanh(z/2)) / 2, so silu(z) = h + h * tanh(h) with h = z/2,
// using the hardware tanh approximation (relative error about 2^-11, below the
// 2^-9 of the bf16 rounding that follows).
__device__ __forceinline__ float silu_tanh(float z) {
  const float h = 0.5f * z;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

// The same as z / (1 + e^-z): two special-function operations (exp and the
// reciprocal of the division).  Kept for comparison (CONV3D_GN_SILU=exp).
__device__ __forceinline__ float silu_exp(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

__device__ __forceinline__ void unpack8(const uint4 q, uint32_t (&e)[8]) {
  e[0] = q.x & 0xFFFFu; e[1] = q.x >> 16; e[2] = q.y & 0xFFFFu; e[3] = q.y >> 16;
  e[4] = q.z & 0xFFFFu; e[5] = q.z >> 16; e[6] = q.w & 0xFFFFu; e[7] = q.w >> 16;
}

// Asynchronous 16-byte copy global -> shared (no registers held while it is
// in flight) and its group bookkeeping.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Pixel rows each thread of the statistics pass keeps in flight.
constexpr int GN_DEPTH = 8;

// Block (v, r): thread (v + vecs * r) owns the 8 channels [8v, 8v+8) of the
// pixels r, r + rows, r + 2 rows, ... of its chunk.  Its 16-byte vectors
// stream through its own GN_DEPTH slots of a shared-memory ring by cp.async,
// GN_DEPTH rows ahead of the one it adds (a thread reads only the slots it
// filled, so no barrier is needed; measured on B200: with four loads held in
// registers instead, the single-set 75 MB tensor streamed at 2.0 TB/s).  Per
// channel it sums (x - K) and (x - K)^2 in fp32 with K = x at the set's first
// pixel (shifting by a sample of the data keeps the fp32 partial sums small).
// The block folds the rows together, expands to {sum x, sum x^2} in fp64 per
// channel, adds the channels of each group in shared memory and issues one
// pair of fp64 atomics per group.
template <bool kBF16>
__global__ void __launch_bounds__(256, 4)
    gn_stats_kernel(const uint16_t* __restrict__ x,
                                                       double* __restrict__ stats, int C,
                                                       int groups, long long set_pixels,
                                                       int chunk_pixels, int chunks_per_set) {
  // the ring [GN_DEPTH][threads] of 16-byte slots while streaming; afterwards
  // [rows][C][2] floats, then [C][2] doubles
  extern __shared__ __align__(16) float red[];
  const int vecs = C / 8;
  const int rows = blockDim.x / vecs;
  const int v = threadIdx.x % vecs;
  const int r = threadIdx.x / vecs;
  const long long set = blockIdx.x / chunks_per_set;
  const long long chunk = blockIdx.x % chunks_per_set;
  const long long p_begin = chunk * chunk_pixels;
  long long p_end = p_begin + chunk_pixels;
  if (p_end > set_pixels) p_end = set_pixels;
  const uint16_t* xs = x + set * set_pixels * C;
  double* csum = reinterpret_cast<double*>(red + static_cast<size_t>(rows) * C * 2);

  float K[8], s1[8], s2[8];
  {
    uint32_t e[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(xs + 8 * v)), e);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      K[j] = to_f<kBF16>(e[j]);
      s1[j] = 0.0f;
      s2[j] = 0.0f;
    }
  }
  // GN_DEPTH rows in flight per thread: with four 8-warp blocks per SM that
  // keeps 128 KB of reads outstanding on every SM
  const long long first = p_begin + r;
  const long long nrow = first < p_end ? (p_end - first + rows - 1) / rows : 0;   // rows of this thread
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(red)) + threadIdx.x * 16u;
  const uint32_t ring_step = blockDim.x * 16u;
  const uint16_t* src = xs + first * C + 8 * v;
  const long long src_step = static_cast<long long>(rows) * C;
#pragma unroll
  for (int k = 0; k < GN_DEPTH; ++k) {
    if (k < nrow) cp_async16(ring + k * ring_step, src + k * src_step);
    cp_async_commit();   // one group per row, empty ones included, so the count stays fixed
  }
  for (long long k = 0; k < nrow; ++k) {
    cp_async_wait<GN_DEPTH - 1>();   // row k has landed
    const uint32_t slot = ring + static_cast<uint32_t>(k % GN_DEPTH) * ring_step;
    uint4 q;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w)
                 : "r"(slot)
                 : "memory");
    uint32_t e[8];
    unpack8(q, e);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float d = to_f<kBF16>(e[j]) - K[j];
      s1[j] += d;
      s2[j] = fmaf(d, d, s2[j]);
    }
    // the slot was read into registers above: refill it with row k + GN_DEPTH
    if (k + GN_DEPTH < nrow) cp_async16(slot, src + (k + GN_DEPTH) * src_step);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();   // every thread's ring slots are drained before red reuses them
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    red[(r * C + 8 * v + j) * 2 + 0] = s1[j];
    red[(r * C + 8 * v + j) * 2 + 1] = s2[j];
  }
  __syncthreads();
  // one thread per channel: fold the rows and expand the shift in fp64
  const double n = static_cast<double>(p_end > p_begin ? p_end - p_begin : 0);
  const int cg = C / groups;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    double a = 0.0, b = 0.0;
    for (int rr = 0; rr < rows; ++rr) {
      a += red[(rr * C + c) * 2 + 0];
      b += red[(rr * C + c) * 2 + 1];
    }
    const double k = to_f<kBF16>(xs[c]);
    // sum x = n k + sum d ; sum x^2 = sum d^2 + 2 k sum d + n k^2
    csum[2 * c + 0] = n * k + a;
    csum[2 * c + 1] = b + 2.0 * k * a + n * k * k;
  }
  __syncthreads();
  // one thread per group: add its channels (in place: group g's sums go to csum[2c0..])
  for (int g = threadIdx.x; g < groups; g += blockDim.x) {
    double a = 0.0, b = 0.0;
    for (int c = g * cg; c < (g + 1) * cg; ++c) {
      a += csum[2 * c + 0];
      b += csum[2 * c + 1];
    }
    // only this thread reads or writes the channels of group g, so the first
    // channel's slot can hold the group's sum
    csum[2 * (g * cg) + 0] = a;
    csum[2 * (g * cg) + 1] = b;
  }
  __syncthreads();
  for (int g = threadIdx.x; g < groups; g += blockDim.x) {
    atomicAdd(&stats[(set * groups + g) * 2 + 0], csum[2 * (g * cg) + 0]);
    atomicAdd(&stats[(set * groups + g) * 2 + 1], csum[2 * (g * cg) + 1]);
  }
}

// {sum, sum of squares} over `count` elements -> {mean, 1/sqrt(var + eps)}.
__global__ void gn_finalize_kernel(double* stats, long long pairs, double count, double eps) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < pairs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const double mu = stats[2 * i] / count;
    double var = stats[2 * i + 1] / count - mu * mu;
    if (var < 0.0) var = 0.0;
    stats[2 * i] = mu;
    stats[2 * i + 1] = 1.0 / sqrt(var + eps);
  }
}

}  // namespace conv3d_gn

// {sum, sum of squares} -> {mean, 1/sqrt(var + eps)} in place, for `pairs`
// statistic entries of `count` values each (used by the convolution that
// gathers its output's statistics in its epilogue).
cudaError_t conv3d_gn_finalize(double* stats, long long pairs, double count, double eps,
                               cudaStream_t stream) {
  conv3d_gn::gn_finalize_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, stream>>>(
      stats, pairs, count, eps);
  return conv3d_count_launches(1);
}

namespace conv3d_gn {

// y = silu((x - mean) * rstd * gamma + beta) (or without the silu).  The grid
// stride is a multiple of C/8 vectors, so each thread keeps the same 8
// channels: their gamma/beta are loaded once and the per-channel scale/shift
// are recomputed only when the thread moves to another statistic set.
template <bool kBF16>
__global__ void __launch_bounds__(256, 3) gn_apply_kernel(const uint16_t* x,
                                                          const double* __restrict__ stats,
                                                          const uint16_t* __restrict__ gamma,
                                                          const uint16_t* __restrict__ beta,
                                                          uint16_t* y, long long pixels, int C,
                                                          int groups, long long set_pixels,
                                                          int apply_silu) {
  const int vecs = C / 8;
  const long long total = pixels * vecs;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= total) return;
  const int c0 = static_cast<int>(i % vecs) * 8;
  const int cg = C / groups;
  const long long pstride = stride / vecs;         // pixels advanced per grid step
  long long p = i / vecs;                          // this thread's current pixel
  long long set_end = -1;                          // first pixel past the cached set
  float scale[8], shift[8];
  // four independent 16-byte loads in flight per thread, then compute and store
  constexpr int U = 4;
  for (; i < total; i += U * stride, p += U * pstride) {
    uint4 q[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i + u * stride < total) q[u] = *reinterpret_cast<const uint4*>(x + (i + u * stride) * 8);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long iu = i + u * stride;
      if (iu >= total) break;
      const long long pu = p + u * pstride;
      if (pu >= set_end || pu < set_end - set_pixels) {
        const long long set = pu / set_pixels;
        set_end = (set + 1) * set_pixels;
        uint32_t ga[8], be[8];
        if (gamma) unpack8(__ldg(reinterpret_cast<const uint4*>(gamma + c0)), ga);
        if (beta) unpack8(__ldg(reinterpret_cast<const uint4*>(beta + c0)), be);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const double* st = stats + (set * groups + (c0 + j) / cg) * 2;
          scale[j] = static_cast<float>(st[1]) * (gamma ? to_f<kBF16>(ga[j]) : 1.0f);
          // one fused multiply-add, as in the convolution's own operand transform
          shift[j] = fmaf(-static_cast<float>(st[0]), scale[j], beta ? to_f<kBF16>(be[j]) : 0.0f);
        }
      }
      uint32_t e[8];
      unpack8(q[u], e);
      float z[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        z[j] = fmaf(to_f<kBF16>(e[j]), scale[j], shift[j]);
        if (apply_silu == 1) z[j] = silu_tanh(z[j]);
        else if (apply_silu == 2) z[j] = silu_exp(z[j]);
      }
      // one two-lane conversion per pair (same round-to-nearest-even as one
      // conversion per value, fewer instructions: measured 929 -> 836 us on a
      // 2 GB tensor)
      uint4 w;
      w.x = pack2<kBF16>(z[0], z[1]);
      w.y = pack2<kBF16>(z[2], z[3]);
      w.z = pack2<kBF16>(z[4], z[5]);
      w.w = pack2<kBF16>(z[6], z[7]);
      *reinterpret_cast<uint4*>(y + iu * 8) = w;
    }
  }
}

conv3d_status_t check_common(const void* x, int N, int D, int H, int W, int C, int groups,
                             conv3d_dtype_t dtype) {
  if (!x || N < 1 || D < 1 || H < 1 || W < 1 || C < 1 || groups < 1) return CONV3D_ERR_INVALID_ARG;
  if (dtype != CONV3D_F16 && dtype != CONV3D_BF16) return CONV3D_ERR_INVALID_ARG;
  if (C % groups != 0) return CONV3D_ERR_INVALID_ARG;
  if (C % 8 != 0 || C > 2048) return CONV3D_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(x) & 15u) return CONV3D_ERR_ALIGNMENT;
  return CONV3D_OK;
}

}  // namespace conv3d_gn

using namespace conv3d_gn;

extern "C" {

conv3d_status_t conv3d_groupnorm_stats(const void* x, int N, int D, int H, int W, int C,
                                       int groups, int per_frame, float eps, conv3d_dtype_t dtype,
                                       double* stats, struct CUstream_st* stream) {
  conv3d_status_t st = check_common(x, N, D, H, W, C, groups, dtype);
  if (st != CONV3D_OK) return st;
  if (!stats || !(eps >= 0.0f)) return CONV3D_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(stats) & 7u) return CONV3D_ERR_ALIGNMENT;
  const long long frame_pixels = static_cast<long long>(H) * W;
  const long long set_pixels = per_frame ? frame_pixels : frame_pixels * D;
  const long long sets = per_frame ? static_cast<long long>(N) * D : N;
  const int vecs = C / 8;
  int rows = 256 / vecs;
  if (rows < 1) rows = 1;
  const int threads = vecs * rows;
  if (threads > 256) return CONV3D_ERR_UNSUPPORTED;   // C <= 2048
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Pixels per block: one resident wave (four blocks per SM) for small
  // tensors, so that few blocks end in a reduction and same-address atomics;
  // at most 1024 for large ones, so that the many waves leave a short tail
  // (measured on B200: 75 MB single set 41 -> 37 us; 2 GB per-frame sets,
  // where 8 blocks per SM rounded up to 2.04 waves, 384 -> 336 us); at
  // least 16 pixels per row of threads.
  long long chunk_pixels = (sets * set_pixels + 4LL * sms - 1) / (4LL * sms);
  if (chunk_pixels > 1024) chunk_pixels = 1024;
  if (chunk_pixels < 16LL * rows) chunk_pixels = 16LL * rows;
  if (const char* env = getenv("CONV3D_GN_CHUNK")) {   // tuning knob: pixels per block
    const long long v = atoll(env);
    if (v > 0) chunk_pixels = v;
  }
  if (chunk_pixels > set_pixels) chunk_pixels = set_pixels;
  long long chunks = (set_pixels + chunk_pixels - 1) / chunk_pixels;

  const long long blocks = sets * chunks;
  if (blocks > 0x7FFFFFFFLL) return CONV3D_ERR_UNSUPPORTED;
  const size_t red_bytes =
      static_cast<size_t>(rows) * C * 2 * sizeof(float) + 2 * C * sizeof(double);
  const size_t ring_bytes = static_cast<size_t>(GN_DEPTH) * threads * 16;
  const size_t smem = red_bytes > ring_bytes ? red_bytes : ring_bytes;
  if (smem > 48 * 1024) return CONV3D_ERR_UNSUPPORTED;
  cudaError_t e = cudaMemsetAsync(stats, 0, sets * groups * 2 * sizeof(double), stream);
  if (e != cudaSuccess) return CONV3D_ERR_CUDA;
  if (dtype == CONV3D_BF16)
    gn_stats_kernel<true><<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        static_cast<const uint16_t*>(x), stats, C, groups, set_pixels,
        static_cast<int>(chunk_pixels), static_cast<int>(chunks));
  else
    gn_stats_kernel<false><<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        static_cast<const uint16_t*>(x), stats, C, groups, set_pixels,
        static_cast<int>(chunk_pixels), static_cast<int>(chunks));
  if (conv3d_count_launches(1) != cudaSuccess) return CONV3D_ERR_CUDA;
  const long long pairs = sets * groups;
  gn_finalize_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, stream>>>(
      stats, pairs, static_cast<double>(set_pixels) * (C / groups), static_cast<double>(eps));
  return conv3d_count_launches(1) == cudaSuccess ? CONV3D_OK : CONV3D_ERR_CUDA;
}

conv3d_status_t conv3d_groupnorm_silu(const void* x, const double* stats, const void* gamma,
                                      const void* beta, void* y, int N, int D, int H, int W,
                                      int C, int groups, int per_frame, int apply_silu,
                                      conv3d_dtype_t dtype, struct CUstream_st* stream) {
  conv3d_status_t st = check_common(x, N, D, H, W, C, groups, dtype);
  if (st != CONV3D_OK) return st;
  if (!stats || !y) return CONV3D_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y) & 15u) || (reinterpret_cast<uintptr_t>(stats) & 7u) ||
      (gamma && (reinterpret_cast<uintptr_t>(gamma) & 15u)) ||
      (beta && (reinterpret_cast<uintptr_t>(beta) & 15u)))
    return CONV3D_ERR_ALIGNMENT;
  const long long pixels = static_cast<long long>(N) * D * H * W;
  const long long frame_pixels = static_cast<long long>(H) * W;
  const long long set_pixels = per_frame ? frame_pixels : frame_pixels * D;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // block size a multiple of C/8 vectors: every thread keeps its 8 channels
  const int vpp = C / 8;
  int threads = (256 / vpp) * vpp;
  if (threads < vpp) threads = vpp;
  if (threads > 256) return CONV3D_ERR_UNSUPPORTED;   // C <= 2048
  const long long vecs = pixels * vpp;
  long long blocks = (vecs + 4LL * threads - 1) / (4LL * threads);
  if (blocks > static_cast<long long>(sms) * 3) blocks = static_cast<long long>(sms) * 3;
  // SiLU form: 1 = tanh (one special-function op, the default), 2 = exp and
  // division (CONV3D_GN_SILU=exp, for comparison)
  if (apply_silu) {
    const char* env = getenv("CONV3D_GN_SILU");
    apply_silu = (env != nullptr && env[0] == 'e') ? 2 : 1;
  }
  if (dtype == CONV3D_BF16)
    gn_apply_kernel<true><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        static_cast<const uint16_t*>(x), stats, static_cast<const uint16_t*>(gamma),
        static_cast<const uint16_t*>(beta), static_cast<uint16_t*>(y), pixels, C, groups,
        set_pixels, apply_silu);
  else
    gn_apply_kernel<false><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        static_cast<const uint16_t*>(x), stats, static_cast<const uint16_t*>(gamma),
        static_cast<const uint16_t*>(beta), static_cast<uint16_t*>(y), pixels, C, groups,
        set_pixels, apply_silu);
  return conv3d_count_launches(1) == cudaSuccess ? CONV3D_OK : CONV3D_ERR_CUDA;
}

}  // extern "C"
