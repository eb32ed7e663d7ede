// wgrad_kernel.cuh -- the weight gradient of the implicit-GEMM convolution,
// dw[co, tap, ci] = sum over output pixels m of dy[m, co] * A[m, (tap, ci)],
// A being the same implicit im2col matrix the forward pass reads (the pages'
// on-device fine-tuning trains convolution layers: engineering.drawthings.ai,
// LoRA post).
//
// As a GEMM the reduction runs over output pixels, which neither x nor dy
// stores innermost, so both tcgen05 operands are MN-major: M = 128 rows of
// (tap, ci) -- one tap, two 64-channel chunks -- and N = up to 256 output
// channels, K = 128 output pixels per pipeline stage (eight K = 16 MMAs).  A
// stage holds two im2col loads (128 pixels x 64 channels) and BN/64 tiled
// loads of dy (128 pixels x 64 channels), each 128 rows of 128 swizzled bytes:
// exactly the MN-major 128-byte-swizzle layout (64-element blocks 16 KB apart
// along M/N, 8-row groups 1 KB apart along K).  128 pixels per stage rather
// than 64 halves the copies and barrier round trips per byte (measured on
// B200: 1290 -> 1608 TFLOP/s on a 256-channel 9x128x128 layer); 32 was far
// slower.  A stage of six boxes (the swapped variant below, one-CTA
// 256-channel tiles) is 96 KB at 128 pixels, so only two fit; those take
// 96-pixel stages, three of them, so that two stages load while one feeds
// the MMAs (kPix, chosen on the host).
//
// A swapped variant serves layers with at most 128 output channels, where an
// N = 128 product would take as long as an N = 256 one: M = 128 output
// channels (dy, two 64-channel boxes) and N = up to 256 (tap, ci) entries --
// four 64-channel im2col boxes of taps that share the temporal offset, so
// every chunk is skipped or used by the whole unit.
//
// A pair variant (cta_group::2, a cluster of two CTAs) computes M = 256:
// CTA r holds the 128 rows of its own (tap, channel block) -- the two blocks
// share the temporal tap -- and half of the 256 output channels of dy, so
// each CTA moves 64 KB per chunk instead of 96 KB for the same products.
//
// Work unit = (tap and 128-channel block, output-channel block, range of
// kPix-pixel chunks), or (temporal tap and block of four entries, ...) when
// swapped, or (temporal tap and pair of blocks, ...) for CTA pairs;
// persistent CTAs (or clusters) walk the units.  Chunks whose temporal tap
// reads zero padding are skipped by producer and MMA alike; chunk rows past
// the frame read dy as zero.  Each finished unit adds its 128 x BN fp32 block
// to a zeroed fp32 gradient with coalesced atomics (one warp: 32 consecutive
// (tap, ci) entries of one output channel per instruction).
#pragma once

#include "conv3d_kernel.cuh"

namespace conv3d {

struct WgradParams {
  int D, Do, Ho, Wo, HoWo;
  int Cin, Cout;
  int kt, kh, kw;
  int st, sh, sw;
  int pf, ph, pw;
  int tpad;                 // 0 zero, 1 causal replicate, 2 causal zero, 3 cached frames
  int taps;
  int cblocks;              // ceil(Cin / 128)                  (plain variant)
  int BN;                   // output channels per unit: multiple of 64, <= 256 (plain), 128 (swap)
  int co_tiles;             // ceil(Cout / BN)
  int c64s;                 // Cin / 64                          (swap variant)
  int ents;                 // kh * kw * Cin / 64 entries per temporal tap (swap)
  int eblocks;              // ceil(ents / ent_per_block)        (swap)
  int ent_per_block;        // entries per block: 4 (N = 256) or 3 (N = 192)  (swap)
  int pairs_per_it;         // ceil(kh * kw * cblocks / 2)       (pair)
  int chunks_per_frame;     // ceil(HoWo / 64)
  long long total_chunks;   // N * Do * chunks_per_frame
  int splits;               // chunk ranges per (tap block, co tile)
  int num_units;
  int stages;
  uint32_t tmem_cols;
  uint32_t acc_cols;        // TMEM columns per accumulator (BN plain, 256 swapped)
  uint32_t idesc;
  float* dw;                // [Cout][taps][Cin] fp32, accumulated
  float* db;                // [Cout] fp32 bias gradient, accumulated (bias block instances)
  int db_it;                // temporal tap whose frame walk the bias block follows
  int* status;
  unsigned long long timeout_ns;
  int test_stall;           // failure-detection test: the producer skips its first stage's copies
};

constexpr int WG_PIX = 128;                         // pixels (K) per stage, by default

// Shared-memory matrix descriptor for an MN-major operand in 64-element x
// 8-row atoms with the 128-byte swizzle: leading byte offset = distance of
// consecutive 64-element blocks along M/N, stride byte offset = distance of
// consecutive 8-row groups along K, version 1, layout type 2.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t mn_block_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((mn_block_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Frame read by temporal tap `it` of output frame `to`: a frame of x (>= 0), a
// cached frame of the previous chunk (-(kt-1) .. -1, cached mode), or kNoFrame
// when the tap reads zero padding.
__device__ __forceinline__ int wg_source_frame(const WgradParams& p, int to, int it) {
  const int f = to * p.st + it - p.pf;
  if (f < 0) return p.tpad == 1 ? 0 : (p.tpad == 3 ? f : kNoFrame);
  return f < p.D ? f : kNoFrame;
}

struct WgUnit {
  int it;            // temporal tap
  int tap, cb;       // plain / pair: tap and 128-channel block of this CTA
  int e0, nent;      // swap: first entry of the block and entries in it (1..ent_per_block)
  bool dup;          // pair: this CTA's block repeats its peer's (odd count): not written
  bool bias;         // the bias block: A = ones, so every row of the product is sum(dy)
  int co0;
  long long c_begin, c_end;
};

template <bool kSwap, bool kPair, bool kBias = false, bool kMix = false>
__device__ __forceinline__ WgUnit wg_decode(const WgradParams& p, int u, uint32_t rank = 0) {
  WgUnit r;
  r.dup = false;
  r.bias = false;
  // split-major: the units that run at the same time share a pixel range, so
  // x and dy come from DRAM about once and serve every tap block from L2
  const int per_split = p.num_units / p.splits;
  const int split = u / per_split;
  const int rest = u - split * per_split;
  const int cot = rest % p.co_tiles;
  const int mb = rest / p.co_tiles;
  if (kPair) {
    // blocks of one temporal tap, (spatial tap, channel block) in order, taken two at a time
    r.it = mb / p.pairs_per_it;
    const int per_it = p.kh * p.kw * p.cblocks;
    int e = 2 * (mb - r.it * p.pairs_per_it) + static_cast<int>(rank);
    if (e >= per_it) {
      e = per_it - 1;
      r.dup = true;
    }
    const int sp = e / p.cblocks;
    r.cb = e - sp * p.cblocks;
    r.tap = r.it * p.kh * p.kw + sp;
    r.e0 = r.nent = 0;
  } else if (kSwap && kMix) {
    // entries numbered across the temporal taps (entry e: tap e / ents), so
    // that only the last block of all may be partly filled
    r.it = 0;
    r.e0 = mb * p.ent_per_block;
    const int all = p.kt * p.ents;
    r.nent = all - r.e0 < p.ent_per_block ? all - r.e0 : p.ent_per_block;
    r.tap = r.cb = 0;
  } else if (kSwap) {
    r.it = mb / p.eblocks;
    r.e0 = (mb - r.it * p.eblocks) * p.ent_per_block;
    r.nent = p.ents - r.e0 < p.ent_per_block ? p.ents - r.e0 : p.ent_per_block;
    r.tap = r.cb = 0;
  } else if (kBias && mb == p.taps * p.cblocks) {
    // one more block per output-channel tile: the bias gradient
    r.bias = true;
    r.tap = r.cb = 0;
    r.it = p.db_it;
    r.e0 = r.nent = 0;
  } else {
    r.tap = mb / p.cblocks;
    r.cb = mb - r.tap * p.cblocks;
    r.it = r.tap / (p.kh * p.kw);
    r.e0 = r.nent = 0;
  }
  r.co0 = cot * p.BN;
  const long long per = (p.total_chunks + p.splits - 1) / p.splits;
  r.c_begin = static_cast<long long>(split) * per;
  if (r.c_begin > p.total_chunks) r.c_begin = p.total_chunks;
  r.c_end = r.c_begin + per < p.total_chunks ? r.c_begin + per : p.total_chunks;
  return r;
}

// Walks a unit's chunk range one output frame at a time: each step yields the
// frame (fo = n*Do + to), the first chunk in it and how many chunks of the
// range it holds.  One division per unit; none per chunk (the issuing threads
// are single threads whose per-chunk cost must stay well under one stage's
// MMA time).
struct FrameWalk {
  long long fo, left;
  int n, to, pc, count;

  __device__ __forceinline__ FrameWalk(const WgradParams& p, const WgUnit& u) {
    fo = u.c_begin / p.chunks_per_frame;
    pc = static_cast<int>(u.c_begin - fo * p.chunks_per_frame);
    n = static_cast<int>(fo / p.Do);
    to = static_cast<int>(fo - static_cast<long long>(n) * p.Do);
    left = u.c_end - u.c_begin;
    count = 0;
  }
  // Advances to the next frame segment; false once the range is exhausted.
  __device__ __forceinline__ bool next(const WgradParams& p) {
    if (count > 0) {
      left -= count;
      pc = 0;
      ++fo;
      if (++to == p.Do) {
        to = 0;
        ++n;
      }
    }
    if (left <= 0) return false;
    const long long room = p.chunks_per_frame - pc;
    count = static_cast<int>(left < room ? left : room);
    return true;
  }
};

// 128-bit fp32 reduction into global memory (four consecutive floats).
__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// kPix = pixels (K) per stage, a multiple of 16: every operand box is kPix
// rows of 128 bytes (64 channels), and the A stage holds two of them.
// kBias: the plain variant with one more block per output-channel tile whose
// A operand is a constant tile of ones in shared memory, so that its product
// is the bias gradient (every row: the sum of dy over the unit's pixels); the
// block loads only dy, which the other blocks of the same pixel range bring
// into L2 at the same time, and its epilogue adds one row to db.
template <bool kBF16, bool kSwap, bool kPair, int kPix, bool kBias = false, bool kMix = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    conv3d_wgrad_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_dy,
                        const __grid_constant__ CUtensorMap map_p, const WgradParams p) {
  static_assert(!(kSwap && kPair), "the pair variant is the plain operand assignment");
  static_assert(!(kBias && (kSwap || kPair)), "the bias block: plain variant only");
  static_assert(!kMix || kSwap, "entry blocks across temporal taps: swapped variant only");
  static_assert(kPix % 16 == 0 && kPix <= 256, "pixels per stage");
  constexpr uint32_t kBox = kPix * 128;          // one 64-channel box
  constexpr uint32_t kABytes = 2 * kBox;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ __align__(8) uint64_t s_peer_bar;      // pairs: the odd CTA's end-of-run report
  __shared__ unsigned long long s_peer_count;
  constexpr int kCtas = kPair ? 2 : 1;
  const uint32_t warp = threadIdx.x / 32;
  const uint32_t lane = threadIdx.x % 32;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int first_unit = blockIdx.x / kCtas;   // this CTA's cluster (or CTA) index
  const int unit_step = gridDim.x / kCtas;

  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  // B operand: dy boxes (plain: BN/64 of them; pair: this CTA's half) or up to
  // four x boxes (swapped)
  const uint32_t b_stage_bytes =
      kSwap ? 4u * kBox : static_cast<uint32_t>(p.BN / kCtas) * kPix * 2;
  const uint32_t a_ring = base;
  const uint32_t b_ring = a_ring + p.stages * kABytes;
  const uint32_t bars = b_ring + p.stages * b_stage_bytes;
  const uint32_t full_bar = bars;
  const uint32_t empty_bar = bars + 8 * p.stages;
  const uint32_t tfull_bar = bars + 16 * p.stages;
  const uint32_t tempty_bar = tfull_bar + 16;
  const uint32_t drain_bar = tempty_bar + 16;
  // bias block: 4 KB of ones, two 64-row blocks (2 KB apart) of 16 pixel rows
  // in the 128-byte-swizzled MN-major layout -- one K = 16 step, reused for
  // every step, as all its values are 1
  const uint32_t ones = (drain_bar + 8 + 1023u) & ~1023u;
  SharedCtl ctl{&s_abort, p.status, p.timeout_ns,
                kPair ? mapa_shared(smem_addr(&s_abort), rank ^ 1u) : 0u};
  const uint32_t peer_bar = smem_addr(&s_peer_bar);
  const uint32_t peer_count = smem_addr(&s_peer_count);

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(peer_bar, 1);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full_bar + 8 * s, 1);
      mbar_init(empty_bar + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar + 8 * a, 1);
      mbar_init(tempty_bar + 8 * a, 4 * kCtas);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_dy);
    if (p.tpad == 3) prefetch_tensormap(&map_p);
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
  if constexpr (kBias) {
    if (warp >= 2) {   // the epilogue warps fill the ones, then make them visible to the MMAs
      const uint32_t one2 = kBF16 ? 0x3F803F80u : 0x3C003C00u;
      for (uint32_t i = threadIdx.x - 64u; i < 1024u; i += NUM_THREADS - 64u)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(ones + 4u * i), "r"(one2) : "memory");
      fence_proxy_async_shared();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();   // the peer's barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      const bool stall = p.test_stall != 0;
      // one CTA's share of a stage (the same for every unit of a pair)
      const uint32_t half_bytes = static_cast<uint32_t>(2 + p.BN / 64 / kCtas) * kBox;
      for (int u = first_unit; ok && u < p.num_units; u += unit_step) {
        const WgUnit wu = wg_decode<kSwap, kPair, kBias, kMix>(p, u, rank);
        // The im2col boxes of the unit: (kw offset, kh offset, first channel).
        // A box whose channels all lie past Cin (or past Cout for dy) is loaded
        // from the unit's first box instead: those rows/columns of the product
        // are never written out, and every copy starts in bounds.
        int bw[4], bh[4], bc[4], bt[4];   // bt: temporal tap of the box (kMix)
        int nx;
        if (kSwap) {
          nx = wu.nent;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            int e = wu.e0 + (j < nx ? j : 0);
            bt[j] = kMix ? e / p.ents : wu.it;
            if (kMix) e -= bt[j] * p.ents;
            const int sp = e / p.c64s;
            bc[j] = (e - sp * p.c64s) * 64;
            bh[j] = sp / p.kw;
            bw[j] = sp - bh[j] * p.kw;
          }
        } else {
          nx = (kBias && wu.bias) ? 0 : 2;   // the bias block loads dy only
          const int sp = wu.tap - wu.it * p.kh * p.kw;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            bh[j] = sp / p.kw;
            bw[j] = sp - bh[j] * p.kw;
            bc[j] = 2 * wu.cb * 64 + (j == 1 && 2 * wu.cb * 64 + 64 < p.Cin ? 64 : 0);
          }
        }
        // dy boxes: the unit's output channels (this CTA's half for a pair) in
        // 64-channel steps
        const int ndy = kSwap ? 2 : p.BN / 64 / kCtas;
        const int dy_c0 = wu.co0 + static_cast<int>(rank) * (p.BN / kCtas);
        const uint32_t x_ring = kSwap ? b_ring : a_ring;
        const uint32_t x_stage = kSwap ? b_stage_bytes : kABytes;
        const uint32_t dy_ring = kSwap ? a_ring : b_ring;
        const uint32_t dy_stage = kSwap ? kABytes : b_stage_bytes;
        const uint32_t tx_bytes = static_cast<uint32_t>(kCtas * (nx + ndy)) * kBox;
        FrameWalk fw(p, wu);
        while (ok && fw.next(p)) {
          const int f = wg_source_frame(p, fw.to, wu.it);
          if (!kMix && f == kNoFrame) continue;   // this tap reads zero padding here
          // frames before the chunk come from the cached-frames tensor
          const CUtensorMap* xmap = f < 0 ? &map_p : &map_x;
          const int img = f < 0 ? fw.n * (p.kt - 1) + (p.kt - 1) + f : fw.n * p.D + f;
          // kMix: each box's own frame; a tap that reads zero padding loads an
          // image index past the tensor, which the copy fills with zeros
          const CUtensorMap* bmap[4];
          int bimg[4];
          if constexpr (kMix) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int fq = wg_source_frame(p, fw.to, bt[q]);
              bmap[q] = fq != kNoFrame && fq < 0 ? &map_p : &map_x;
              bimg[q] = fq == kNoFrame ? -1
                        : fq < 0       ? fw.n * (p.kt - 1) + (p.kt - 1) + fq
                                       : fw.n * p.D + fq;
            }
          }
          int p0 = fw.pc * kPix;
          int ho0 = p0 / p.Wo;
          int wo0 = p0 - ho0 * p.Wo;
          for (int j = 0; j < fw.count; ++j) {
            if (!wait_bounded(empty_bar + 8 * stage, phase ^ 1, ctl, true)) {
              ok = false;
              break;
            }
            const uint32_t fb = full_bar + 8 * stage;
            const uint32_t x_dst = x_ring + stage * x_stage;
            const uint32_t dy_dst = dy_ring + stage * dy_stage;
            const int wx = wo0 * p.sw - p.pw, hx = ho0 * p.sh - p.ph;
            if (stall && issued == 0) {
              // failure-detection test: this stage never fills, so the
              // tensor-core issuer's wait on it must run out
            } else if constexpr (kPair) {
              if (leader) mbar_arrive_expect_tx(fb, tx_bytes);
              // both CTAs' copies complete on the even CTA's barrier
              const uint32_t fb0 = mapa_shared(fb, 0);
#pragma unroll
              for (int q = 0; q < 2; ++q)
                tma_load_im2col_4d_pair(x_dst + q * kBox, xmap, fb0, bc[q], wx, hx,
                                        img, static_cast<uint16_t>(bw[q]),
                                        static_cast<uint16_t>(bh[q]));
              for (int q = 0; q < ndy; ++q) {
                const int dc = dy_c0 + 64 * q < p.Cout ? dy_c0 + 64 * q : wu.co0;
                tma_load_3d_pair(dy_dst + q * kBox, &map_dy, fb0, dc, p0,
                                 static_cast<int>(fw.fo));
              }
            } else {
              mbar_arrive_expect_tx(fb, tx_bytes);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (q < nx)
                  tma_load_im2col_4d(x_dst + q * kBox, kMix ? bmap[q] : xmap, fb, bc[q], wx, hx,
                                     kMix ? bimg[q] : img, static_cast<uint16_t>(bw[q]),
                                     static_cast<uint16_t>(bh[q]));
              for (int q = 0; q < ndy; ++q) {
                const int dc = dy_c0 + 64 * q < p.Cout ? dy_c0 + 64 * q : wu.co0;
                tma_load_3d(dy_dst + q * kBox, &map_dy, fb, dc, p0,
                            static_cast<int>(fw.fo));
              }
            }
            ++issued;
            if (++stage == static_cast<uint32_t>(p.stages)) {
              stage = 0;
              phase ^= 1;
            }
            p0 += kPix;
            wo0 += kPix;
            while (wo0 >= p.Wo) {
              wo0 -= p.Wo;
              ++ho0;
            }
          }
        }
      }
      producer_finish<kPair>(!ok, issued, stall, p.stages, full_bar, half_bytes, peer_count,
                             peer_bar, ctl, leader);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int local = 0;
      // descriptors of stage 0; a stage or a K step moves the start address
      // (bits 0-13, in 16-byte units) only
      const uint64_t da0 = smem_desc_mn_sw128(a_ring, kBox);
      const uint64_t db0 = smem_desc_mn_sw128(b_ring, kBox);
      const uint64_t d_ones = smem_desc_mn_sw128(ones, 2048);   // bias block: the same K step each time
      for (int u = first_unit; ok && u < p.num_units; u += unit_step, ++local) {
        const WgUnit wu = wg_decode<kSwap, kPair, kBias, kMix>(p, u);
        // swapped: N = 64 per entry of the block
        const uint32_t idesc =
            kSwap ? (p.idesc & ~(0x3Fu << 17)) | (static_cast<uint32_t>(wu.nent * 64 >> 3) << 17)
                  : p.idesc;
        const uint32_t acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!wait_bounded(tempty_bar + 8 * acc, acc_phase ^ 1, ctl, true)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(p.acc_cols);
        uint32_t accumulate = 0;
        FrameWalk fw(p, wu);
        while (ok && fw.next(p)) {
          if (!kMix && wg_source_frame(p, fw.to, wu.it) == kNoFrame) continue;
          for (int j = 0; j < fw.count; ++j) {
            if (!wait_bounded(full_bar + 8 * stage, phase, ctl, true)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = da0 + ((stage * kABytes) >> 4);
            const uint64_t db = db0 + ((stage * b_stage_bytes) >> 4);
            const bool ones_a = kBias && wu.bias;
#pragma unroll
            for (int k = 0; k < kPix / 16; ++k) {
              // 16 pixels = two 8-row groups (2 KB) further along K
              if constexpr (kPair)
                mma_f16_ss_pair(d_tmem, da + k * (2048 >> 4), db + k * (2048 >> 4), idesc,
                                accumulate);
              else
                mma_f16_ss(d_tmem, ones_a ? d_ones : da + k * (2048 >> 4), db + k * (2048 >> 4),
                           idesc, accumulate);
              accumulate = 1;
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
        }
        if (!ok) break;
        if constexpr (kPair) {
          mma_commit_pair(tfull_bar + 8 * acc);
          mma_commit_pair(mapa_shared(tfull_bar + 8 * acc, 1));
        } else {
          mma_commit(tfull_bar + 8 * acc);
        }
      }
      if constexpr (kPair)
        mma_commit_pair(drain_bar);
      else
        mma_commit(drain_bar);
      wait_bounded(drain_bar, 0, ctl, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Plain: thread = one (tap, ci) row of the unit (TMEM lane), 32 output
    // channels per TMEM load; fp32 atomic adds into dw[co][tap][ci], one
    // warp-wide instruction covering 32 consecutive ci of one co (128 bytes).
    // Swapped: thread = one output channel, 32 consecutive ci of one entry per
    // TMEM load, added with eight 16-byte reductions.
    // Launched as a programmatic dependent of the kernel that clears the fp32
    // accumulators: only these warps touch them, so only they wait for it
    // (long before their first unit's MMAs are done); the producer streams x
    // and dy, which the work before the clear wrote, from the start.
    griddep_wait();
    const uint32_t quarter = warp & 3;
    int local = 0;
    const long long K = static_cast<long long>(p.taps) * p.Cin;
    for (int u = first_unit; u < p.num_units; u += unit_step, ++local) {
      const uint32_t acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!wait_bounded(tfull_bar + 8 * acc, acc_phase, ctl, true)) break;
      tc_fence_after();
      const WgUnit wu = wg_decode<kSwap, kPair, kBias, kMix>(p, u, rank);
      // a unit whose chunks all read zero padding issued no MMA: nothing to add
      bool any = false;
      FrameWalk fw(p, wu);
      while (!any && fw.next(p)) any = kMix || wg_source_frame(p, fw.to, wu.it) != kNoFrame;
      const uint32_t t_row =
          tmem_base + ((quarter * 32u) << 16) + acc * static_cast<uint32_t>(p.acc_cols);
      if (kSwap) {
        const int co = wu.co0 + static_cast<int>(quarter * 32 + lane);
        const bool row_ok = any && co < p.Cout;
        for (int j = 0; j < 2 * wu.nent; ++j) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + j * 32, r);
          tmem_ld_wait();
          if (row_ok) {
            int e = wu.e0 + j / 2;
            const int it = kMix ? e / p.ents : wu.it;
            if (kMix) e -= it * p.ents;
            const int sp = e / p.c64s;
            const int tap = it * p.kh * p.kw + sp;
            const int ci0 = (e - sp * p.c64s) * 64 + (j & 1) * 32;
            float* dst = p.dw + static_cast<long long>(co) * K +
                         static_cast<long long>(tap) * p.Cin + ci0;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              red_add_v4(dst + 4 * q, __uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                         __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          }
        }
      } else if (kBias && wu.bias) {
        // every row of the bias block holds sum(dy): row 0 (lane 0 of the
        // first quarter) is added to db, 16 bytes at a time
        if (quarter == 0) {
          for (int j = 0; j < p.BN / 32; ++j) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + j * 32, r);
            tmem_ld_wait();
            const int c0 = wu.co0 + j * 32;
            if (any && lane == 0) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (c0 + 4 * q < p.Cout)
                  red_add_v4(p.db + c0 + 4 * q, __uint_as_float(r[4 * q]),
                             __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                             __uint_as_float(r[4 * q + 3]));
            }
          }
        }
      } else {
        const int ci = wu.cb * 128 + static_cast<int>(quarter * 32 + lane);
        const bool row_ok = any && !wu.dup && ci < p.Cin;
        float* dst = p.dw + static_cast<long long>(wu.co0) * K +
                     static_cast<long long>(wu.tap) * p.Cin + ci;
        for (int j = 0; j < p.BN / 32; ++j) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + j * 32, r);
          tmem_ld_wait();
          if (row_ok) {
            const int co_left = p.Cout - (wu.co0 + j * 32);
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < co_left) atomicAdd(dst + static_cast<long long>(j * 32 + e) * K,
                                         __uint_as_float(r[e]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair)
          mbar_arrive_cluster(mapa_shared(tempty_bar + 8 * acc, 0));
        else
          mbar_arrive(tempty_bar + 8 * acc);
      }
    }
  }

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

// 8 fp32 values -> 8 rounded 16-bit ones (16 bytes).
template <bool kBF16>
__device__ __forceinline__ uint4 round8(const float* __restrict__ src) {
  using C = Cvt<kBF16>;
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  return make_uint4(C::pack(a.x, a.y), C::pack(a.z, a.w), C::pack(b.x, b.y), C::pack(b.z, b.w));
}

// Clears n4 16-byte words at p.  The weight-gradient kernel that follows it
// on the stream may start at once (programmatic launch): only its epilogue
// waits for this grid.
__global__ void zero_f32x4_kernel(float4* __restrict__ p, long long n4) {
  griddep_launch_dependents();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

// fp32 accumulation -> the 16-bit weight gradient (one rounding); the n2
// values of a second array (the bias gradient) in the same launch.  8 values
// per thread: n and n2 are multiples of 8 and every pointer 16-byte aligned.
template <bool kBF16>
__global__ void f32_to_16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst,
                                 long long n, const float* __restrict__ src2 = nullptr,
                                 uint16_t* __restrict__ dst2 = nullptr, long long n2 = 0) {
  griddep_wait();   // (a programmatic dependent of the weight-gradient kernel)
  const long long v1 = n / 8, v = v1 + n2 / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < v;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (i < v1)
      reinterpret_cast<uint4*>(dst)[i] = round8<kBF16>(src + 8 * i);
    else
      reinterpret_cast<uint4*>(dst2)[i - v1] = round8<kBF16>(src2 + 8 * (i - v1));
  }
}

// The same rounding, written to each of kt equal temporal taps:
// dst[co][it][s] = src[co][s] for s < per_co (kh * kw * Cin entries, a
// multiple of 8), 8 values per thread.
template <bool kBF16>
__global__ void f32_to_16_bcast_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst,
                                       int Cout, int kt, long long per_co) {
  griddep_wait();   // (a programmatic dependent of the weight-gradient kernel)
  const long long v = static_cast<long long>(Cout) * kt * per_co / 8;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < v;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = 8 * i;
    const long long co = e / (kt * per_co);
    const long long s = e % per_co;
    reinterpret_cast<uint4*>(dst)[i] = round8<kBF16>(src + co * per_co + s);
  }
}

// dbias[co] += sum over pixels of dy[m, co], with no shared memory, so that its
// blocks fit beside a weight-gradient CTA on every SM and the two run at once.
// Block = 8 warps over a slab of pixels and up to 256 channels (blockIdx.y
// picks the group); lane = 8 v + r of warp w covers the 16-byte vector
// (8 channels) 4w + v of pixel rows r, r + 8, ... of the slab, eight loads in
// flight (a warp reads 64 contiguous bytes of each of eight rows).  The eight
// row lanes are added with shuffles, then lanes r = 0 add their 8 sums to db
// with two 16-byte reductions.
constexpr int BIAS_THREADS = 256;
constexpr int BIAS_CHANNELS = 256;

template <bool kBF16>
__global__ void __launch_bounds__(BIAS_THREADS) bias_grad_kernel(
    const uint16_t* __restrict__ dy, float* __restrict__ db, long long pixels, int Cout,
    long long pixels_per_block) {
  using C = Cvt<kBF16>;
  const int lane = threadIdx.x & 31;
  const int vec = 4 * (threadIdx.x >> 5) + (lane >> 3);    // 16-byte vector of the group
  const int r = lane & 7;
  const int c = blockIdx.y * BIAS_CHANNELS + 8 * vec;      // first channel of the vector
  const bool live = c < Cout;
  const long long p_begin = blockIdx.x * pixels_per_block;
  long long p_end = p_begin + pixels_per_block;
  if (p_end > pixels) p_end = pixels;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (live) {
    const long long stride = Cout / 8;                     // 16-byte vectors per pixel
    const uint4* src = reinterpret_cast<const uint4*>(dy) + c / 8;
    long long p = p_begin + r;
    for (; p + 56 < p_end; p += 64) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = __ldg(src + (p + 8 * u) * stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc[0] += C::lo(q[u].x); acc[1] += C::hi(q[u].x);
        acc[2] += C::lo(q[u].y); acc[3] += C::hi(q[u].y);
        acc[4] += C::lo(q[u].z); acc[5] += C::hi(q[u].z);
        acc[6] += C::lo(q[u].w); acc[7] += C::hi(q[u].w);
      }
    }
    for (; p < p_end; p += 8) {
      const uint4 q = __ldg(src + p * stride);
      acc[0] += C::lo(q.x); acc[1] += C::hi(q.x); acc[2] += C::lo(q.y); acc[3] += C::hi(q.y);
      acc[4] += C::lo(q.z); acc[5] += C::hi(q.z); acc[6] += C::lo(q.w); acc[7] += C::hi(q.w);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], 1);
    acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], 2);
    acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], 4);
  }
  if (live && r == 0) {
    red_add_v4(db + c, acc[0], acc[1], acc[2], acc[3]);
    red_add_v4(db + c + 4, acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace conv3d
