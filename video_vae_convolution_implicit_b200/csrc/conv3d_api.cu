// conv3d_api.cu -- the C ABI of libconv3d (declared in include/conv3d.h):
// argument validation, problem -> GEMM mapping, tensor-map encoding, the
// first-frame weight fold and the kernel launch.  No call synchronises except
// conv3d_poll_status and the self test; nothing allocates except the cached
// per-stream workspace of conv3d_fwd (first-frame fold, tail-split partials).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "conv3d.h"
#include "conv3d_kernel.cuh"
#include "wgrad_kernel.cuh"

// GroupNorm finalize (groupnorm.cu): {sum, sum of squares} -> {mean, rstd}.
cudaError_t conv3d_gn_finalize(double* stats, long long pairs, double count, double eps,
                               cudaStream_t stream);

// Kernel launches this library has issued in the process (every device and
// stream), counted at enqueue; conv3d_kernel_launches() reads it.
std::atomic<unsigned long long> g_kernel_launches{0};

// The status of `n` launches just enqueued by the GroupNorm kernels'
// translation unit, which it also counts.
cudaError_t conv3d_count_launches(int n) {
  g_kernel_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed);
  return cudaGetLastError();
}

namespace {

using namespace conv3d;

// The status of the `n` launches just enqueued, which it also counts.
cudaError_t launched(int n = 1) { return conv3d_count_launches(n); }

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

thread_local char g_last_error[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
}

conv3d_status_t cuda_fail(cudaError_t e, const char* what) {
  set_error("%s: %s", what, cudaGetErrorString(e));
  return CONV3D_ERR_CUDA;
}

// CONV3D_LOG=1: one line per kernel launch on stderr with the plan chosen for
// it (variant, tiles, grid, pipeline depth), read once per process.
bool plan_log() {
  static const bool on = [] {
    const char* env = getenv("CONV3D_LOG");
    return env != nullptr && env[0] == '1';
  }();
  return on;
}

// Failure-detection test hook (conv3d_test_arm_stall): the number of
// convolution-kernel launches still armed and their wait limit.
std::atomic<int> g_stall_launches{0};
std::atomic<int> g_stall_timeout_ms{50};

// True, consuming one armed launch, if this launch is to stall; sets its limit.
bool take_stall(unsigned long long& timeout_ns) {
  int n = g_stall_launches.load();
  while (n > 0) {
    if (g_stall_launches.compare_exchange_weak(n, n - 1)) {
      timeout_ns = static_cast<unsigned long long>(g_stall_timeout_ms.load()) * 1000000ull;
      return true;
    }
  }
  return false;
}

// ------------------------------------------------------------------ problem

struct Problem {
  int N, Cin, D, H, W, Cout;
  int kt, kh, kw;
  int pt, ph, pw;
  int st, sh, sw;
  int pf, pb;
  int Do, Ho, Wo;
  conv3d_tpad_t tpad;
  conv3d_dtype_t dtype;
  bool has_residual;
  bool out_f32;      // write y in fp32 (internal: the backward pass's padded-frame gradient)
  // mixed output (internal: the data gradient under causal replicate padding):
  // output frames 0 .. f32_frames-1 of each sample, the fp32 parts of dx
  // frame 0, go to f32_out ([N][f32_frames][Ho][Wo][Cout]); frame to >=
  // f32_frames is frame to - f32_frames + 1 of y ([N][y_frames][Ho][Wo][Cout])
  int f32_frames;
  int y_frames;
  void* f32_out;
  // combined front (internal: the data gradient under causal replicate
  // padding): output frame 0 also sums the taps of the combine-1 virtual
  // frames before it (0: off)
  int combine;
  const void* prev;  // cached frames before the chunk (CONV3D_TPAD_CAUSAL_CACHED) or null
  bool fold;  // first-frame path: fold the temporal taps into a (hi, lo) pair
  // first frame with the lo part in e5m2: lo weights w8 ([Cout][kh*kw][Cin],
  // scaled by 2^8) and x8 (x scaled by 2^-8), both one byte a value
  bool lo8;
  const void* x8;
  const void* w8;
  // GroupNorm + SiLU applied to x as it is read (conv3d_fwd_gn); gn_stats null otherwise
  const double* gn_stats;
  const void* gn_gamma;
  const void* gn_beta;
  int gn_groups, gn_per_frame, gn_silu;
  double* gn_out;      // sums of y's GroupNorm statistics (per sample), or null
  int gn_out_groups;
  // data-gradient phases of a strided convolution: the im2col window box is
  // sized for exactly Ho x Wo outputs (front pads ph, pw; stride 1), and the
  // outputs go to strided positions of y_scatter (see KernelParams)
  bool exact_out;
  uint16_t* y_scatter;
  int sc_sh, sc_sw, sc_rh, sc_rw, sc_H, sc_W;
};

bool output_extents(int D, int H, int W, const int k[3], const int stride[3], const int pad[3],
                    conv3d_tpad_t tpad, int& pf, int& pb, int out[3]) {
  if (tpad == CONV3D_TPAD_ZERO) {
    pf = pad[0];
    pb = pad[0];
  } else {
    pf = k[0] - 1;
    pb = 0;
  }
  long long nd = static_cast<long long>(D) + pf + pb - k[0];
  long long nh = static_cast<long long>(H) + 2LL * pad[1] - k[1];
  long long nw = static_cast<long long>(W) + 2LL * pad[2] - k[2];
  if (nd < 0 || nh < 0 || nw < 0) return false;
  out[0] = static_cast<int>(nd / stride[0] + 1);
  out[1] = static_cast<int>(nh / stride[1] + 1);
  out[2] = static_cast<int>(nw / stride[2] + 1);
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

conv3d_status_t validate(const void* x, const void* w, const void* bias, const void* residual,
                         const void* y, int N, int Cin, int D, int H, int W, int Cout,
                         const int kernel[3], const int stride[3], const int pad[3],
                         conv3d_tpad_t tpad, conv3d_dtype_t dtype, Problem& P,
                         const void* prev = nullptr) {
  if (!x || !w || !y || !kernel || !stride || !pad) {
    set_error("x, w, y, kernel, stride and pad must be non-null");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (N < 1 || Cin < 1 || D < 1 || H < 1 || W < 1 || Cout < 1) {
    set_error("sizes must be >= 1");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (dtype != CONV3D_F16 && dtype != CONV3D_BF16) {
    set_error("unknown dtype %d", static_cast<int>(dtype));
    return CONV3D_ERR_INVALID_ARG;
  }
  if (tpad != CONV3D_TPAD_ZERO && tpad != CONV3D_TPAD_CAUSAL_REPLICATE &&
      tpad != CONV3D_TPAD_CAUSAL_ZERO && tpad != CONV3D_TPAD_CAUSAL_CACHED) {
    set_error("unknown temporal padding mode %d", static_cast<int>(tpad));
    return CONV3D_ERR_INVALID_ARG;
  }
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED && kernel && kernel[0] > 1 && !prev) {
    set_error("the cached-frames mode needs the previous frames (conv3d_fwd_cached)");
    return CONV3D_ERR_INVALID_ARG;
  }
  for (int i = 0; i < 3; ++i) {
    if (kernel[i] < 1 || stride[i] < 1 || pad[i] < 0) {
      set_error("kernel and stride must be >= 1 and pad >= 0");
      return CONV3D_ERR_INVALID_ARG;
    }
  }
  if (tpad != CONV3D_TPAD_ZERO && pad[0] != 0) {
    set_error("pad[0] must be 0 for the causal temporal modes");
    return CONV3D_ERR_INVALID_ARG;
  }
  int out[3];
  int pf = 0, pb = 0;
  if (!output_extents(D, H, W, kernel, stride, pad, tpad, pf, pb, out)) {
    set_error("the padded input is smaller than the kernel");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (stride[0] > 8 || stride[1] > 8 || stride[2] > 8) {
    set_error("strides must be <= 8 (the TMA traversal-stride limit)");
    return CONV3D_ERR_UNSUPPORTED;
  }
  for (int i = 0; i < 3; ++i) {
    if (kernel[i] > 8 || pad[i] > 127) {
      set_error("kernel extents must be <= 8 and pads <= 127");
      return CONV3D_ERR_UNSUPPORTED;
    }
  }
  if (Cin % 8 != 0 || Cout % 8 != 0) {
    set_error("Cin and Cout must be multiples of 8 (got %d, %d)", Cin, Cout);
    return CONV3D_ERR_UNSUPPORTED;
  }
  const long long frames = static_cast<long long>(N) * D;
  const long long M = static_cast<long long>(N) * out[0] * out[1] * out[2];
  const long long HoWo = static_cast<long long>(out[1]) * out[2];
  const long long tiles = static_cast<long long>(N) * out[0] * ((HoWo + BM - 1) / BM) *
                          ((Cout + 255) / 256);
  if (frames > 0x7FFFFFFFLL || HoWo > 0x7FFFFFFFLL || tiles > 0x7FFFFFFFLL ||
      static_cast<long long>(H) * W > 0x7FFFFFFFLL) {
    set_error("problem too large for 32-bit tile indexing");
    return CONV3D_ERR_UNSUPPORTED;
  }
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (bias && !aligned16(bias)) ||
      (residual && !aligned16(residual)) || (prev && !aligned16(prev))) {
    set_error("tensor pointers must be 16-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const size_t xb = static_cast<size_t>(frames) * H * W * Cin * 2;
  const size_t wb = static_cast<size_t>(Cout) * kernel[0] * kernel[1] * kernel[2] * Cin * 2;
  const size_t yb = static_cast<size_t>(M) * Cout * 2;
  if (overlaps(y, yb, x, xb) || overlaps(y, yb, w, wb) || overlaps(y, yb, bias, Cout * 2ull)) {
    set_error("y must not overlap x, w or bias");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (residual && residual != y && overlaps(y, yb, residual, yb)) {
    set_error("residual must be exactly y or not overlap it");
    return CONV3D_ERR_INVALID_ARG;
  }
  const size_t pb_bytes = static_cast<size_t>(N) * (kernel[0] - 1) * H * W * Cin * 2;
  if (prev && overlaps(y, yb, prev, pb_bytes)) {
    set_error("y must not overlap prev");
    return CONV3D_ERR_INVALID_ARG;
  }
  P.N = N; P.Cin = Cin; P.D = D; P.H = H; P.W = W; P.Cout = Cout;
  P.kt = kernel[0]; P.kh = kernel[1]; P.kw = kernel[2];
  P.pt = pad[0]; P.ph = pad[1]; P.pw = pad[2];
  P.st = stride[0]; P.sh = stride[1]; P.sw = stride[2];
  P.pf = pf; P.pb = pb;
  P.Do = out[0]; P.Ho = out[1]; P.Wo = out[2];
  P.tpad = tpad;
  P.dtype = dtype;
  P.has_residual = residual != nullptr;
  P.out_f32 = false;
  P.prev = tpad == CONV3D_TPAD_CAUSAL_CACHED ? prev : nullptr;
  // a single causal-replicate frame: every temporal tap of the one output
  // frame reads frame 0 (whatever the temporal stride)
  P.fold = (tpad == CONV3D_TPAD_CAUSAL_REPLICATE && D == 1 && kernel[0] > 1);
  P.gn_stats = nullptr;
  P.gn_gamma = P.gn_beta = nullptr;
  P.gn_groups = P.gn_per_frame = P.gn_silu = 0;
  P.gn_out = nullptr;
  P.gn_out_groups = 0;
  P.exact_out = false;
  P.y_scatter = nullptr;
  P.f32_frames = 0;
  P.y_frames = 0;
  P.f32_out = nullptr;
  P.combine = 0;
  P.lo8 = false;
  P.x8 = nullptr;
  P.w8 = nullptr;
  P.sc_sh = P.sc_sw = 1;
  P.sc_rh = P.sc_rw = 0;
  P.sc_H = P.sc_W = 0;
  return CONV3D_OK;
}

// The folded weight holds a high and a low 16-bit part per element.
size_t fold_bytes(int Cin, int Cout, const int k[3]) {
  const size_t b = 2 * static_cast<size_t>(Cout) * k[1] * k[2] * Cin * 2;
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Scratch of the first frame with the lo part in e5m2: the 16-bit hi weight,
// the 8-bit lo weight, then the 8-bit copy of x (N frames).
size_t lo8_hi_bytes(const Problem& P) {
  return align256(static_cast<size_t>(P.Cout) * P.kh * P.kw * P.Cin * 2);
}
size_t lo8_w8_bytes(const Problem& P) {
  return align256(static_cast<size_t>(P.Cout) * P.kh * P.kw * P.Cin);
}
size_t lo8_bytes(const Problem& P) {
  return lo8_hi_bytes(P) + lo8_w8_bytes(P) +
         align256(static_cast<size_t>(P.N) * P.H * P.W * P.Cin);
}

// CONV3D_LO8=1: the first frame's lo product in e5m2 (conv3d_fwd only).
// Off by default: measured on B200 on a 256->256 256x256 first frame, the
// main kernel went from 119 to 108 us, but converting x to e5m2 takes 8.5 us
// more and the call was slower (127 against 114 us): the 8-bit k-blocks move
// as many bytes as 16-bit ones and ran at 1.2x, not 2x, their rate.
bool lo8_enabled() {
  const char* env = getenv("CONV3D_LO8");
  return env != nullptr && env[0] == '1';
}

// ------------------------------------------------------------------ driver entry points

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
PFN_cuTensorMapEncodeIm2col_v12000 g_encode_im2col = nullptr;
std::once_flag g_entry_once;
cudaError_t g_entry_err = cudaSuccess;

conv3d_status_t load_entry_points() {
  std::call_once(g_entry_once, [] {
    cudaDriverEntryPointQueryResult q1, q2;
    void* p1 = nullptr;
    void* p2 = nullptr;
    cudaError_t e1 = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p1, cudaEnableDefault, &q1);
    cudaError_t e2 = cudaGetDriverEntryPoint("cuTensorMapEncodeIm2col", &p2, cudaEnableDefault, &q2);
    if (e1 != cudaSuccess || q1 != cudaDriverEntryPointSuccess || !p1) {
      g_entry_err = e1 != cudaSuccess ? e1 : cudaErrorNotSupported;
    } else if (e2 != cudaSuccess || q2 != cudaDriverEntryPointSuccess || !p2) {
      g_entry_err = e2 != cudaSuccess ? e2 : cudaErrorNotSupported;
    } else {
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p1);
      g_encode_im2col = reinterpret_cast<PFN_cuTensorMapEncodeIm2col_v12000>(p2);
    }
  });
  if (!g_encode_tiled || !g_encode_im2col) return cuda_fail(g_entry_err, "driver entry points");
  return CONV3D_OK;
}

// ------------------------------------------------------------------ tensor-map cache

// A tensor map is a pure function of its encode arguments (address, sizes,
// strides, box, traversal, swizzle), so a call that repeats an earlier call's
// pointers and shape could reuse the maps encoded then instead of asking the
// driver again (3-5 encodes per launch).  Measured on B200, host time per
// conv3d_fwd call with / without this cache: 4.79 / 4.53 us (the small fp16
// layer), 3.34 / 3.17 us (the 256-channel layer) -- the driver's encode is
// cheaper than building and hashing the key -- so it is off unless
// CONV3D_MAP_CACHE=1.  Keyed by the raw argument bytes; at most
// kMapCacheEntries maps are kept (the cache is emptied when full) and
// conv3d_release empties it.
constexpr size_t kMapCacheEntries = 1024;
std::mutex g_map_mu;
std::unordered_map<std::string, CUtensorMap> g_map_cache;

// CONV3D_MAP_CACHE=1 turns the cache on.
bool map_cache_on() {
  static const bool on = [] {
    const char* env = getenv("CONV3D_MAP_CACHE");
    return env != nullptr && env[0] == '1';
  }();
  return on;
}

template <typename T>
void key_add(std::string& k, const T* v, size_t n) {
  k.append(reinterpret_cast<const char*>(v), sizeof(T) * n);
}

bool map_cache_get(const std::string& key, CUtensorMap& out) {
  std::lock_guard<std::mutex> lock(g_map_mu);
  auto it = g_map_cache.find(key);
  if (it == g_map_cache.end()) return false;
  out = it->second;
  return true;
}

void map_cache_put(const std::string& key, const CUtensorMap& m) {
  std::lock_guard<std::mutex> lock(g_map_mu);
  if (g_map_cache.size() >= kMapCacheEntries) g_map_cache.clear();
  g_map_cache.emplace(key, m);
}

CUresult encode_tiled_cached(CUtensorMap* map, CUtensorMapDataType dt, cuuint32_t rank, void* base,
                             const cuuint64_t* dims, const cuuint64_t* strides,
                             const cuuint32_t* box, const cuuint32_t* estr,
                             CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                             CUtensorMapL2promotion l2, CUtensorMapFloatOOBfill oob) {
  if (!map_cache_on())
    return g_encode_tiled(map, dt, rank, base, dims, strides, box, estr, il, sw, l2, oob);
  std::string key(1, 'T');
  const int e[6] = {static_cast<int>(dt), static_cast<int>(rank), static_cast<int>(il),
                    static_cast<int>(sw), static_cast<int>(l2), static_cast<int>(oob)};
  key_add(key, e, 6);
  key_add(key, &base, 1);
  key_add(key, dims, rank);
  key_add(key, strides, rank - 1);
  key_add(key, box, rank);
  key_add(key, estr, rank);
  if (map_cache_get(key, *map)) return CUDA_SUCCESS;
  CUresult r = g_encode_tiled(map, dt, rank, base, dims, strides, box, estr, il, sw, l2, oob);
  if (r == CUDA_SUCCESS) map_cache_put(key, *map);
  return r;
}

CUresult encode_im2col_cached(CUtensorMap* map, CUtensorMapDataType dt, cuuint32_t rank,
                              void* base, const cuuint64_t* dims, const cuuint64_t* strides,
                              const int* lower, const int* upper, cuuint32_t channels,
                              cuuint32_t pixels, const cuuint32_t* estr, CUtensorMapInterleave il,
                              CUtensorMapSwizzle sw, CUtensorMapL2promotion l2,
                              CUtensorMapFloatOOBfill oob) {
  if (!map_cache_on())
    return g_encode_im2col(map, dt, rank, base, dims, strides, lower, upper, channels, pixels,
                           estr, il, sw, l2, oob);
  std::string key(1, 'I');
  const int e[8] = {static_cast<int>(dt), static_cast<int>(rank), static_cast<int>(il),
                    static_cast<int>(sw), static_cast<int>(l2), static_cast<int>(oob),
                    static_cast<int>(channels), static_cast<int>(pixels)};
  key_add(key, e, 8);
  key_add(key, &base, 1);
  key_add(key, dims, rank);
  key_add(key, strides, rank - 1);
  key_add(key, lower, rank - 2);
  key_add(key, upper, rank - 2);
  key_add(key, estr, rank);
  if (map_cache_get(key, *map)) return CUDA_SUCCESS;
  CUresult r = g_encode_im2col(map, dt, rank, base, dims, strides, lower, upper, channels, pixels,
                               estr, il, sw, l2, oob);
  if (r == CUDA_SUCCESS) map_cache_put(key, *map);
  return r;
}

// ------------------------------------------------------------------ per-device state

struct DeviceState {
  bool init = false;
  int num_sms = 0;
  int max_smem_optin = 0;
  int* status = nullptr;         // address of g_status on this device
  // conv3d_fwd's cached scratch, one buffer per stream it was called on: the
  // first-frame folded weight and the tail split's partials and tickets
  struct Scratch {
    cudaStream_t stream;
    void* ptr;
    size_t bytes;
    unsigned int gen;            // launch generation of the split tickets
  };
  Scratch scratch[16] = {};
  int n_scratch = 0;
  bool attr_set[2048] = {};      // per kernel instance: variant + 8 * features (< 256)
  int pair_clusters = 0;         // co-resident CTA pairs (occupancy query)
  int wg_pair_clusters = 0;      // the same for the weight-gradient kernel
  bool wg_attr_set[32] = {};     // per weight-gradient kernel variant (5 kinds x pix x dtype)
  // Second stream (highest priority) on which the data gradient's front frames
  // run beside its body; created on first use, never if creation fails.
  cudaStream_t aux = nullptr;
  cudaEvent_t aux_fork = nullptr, aux_join = nullptr;
  bool aux_failed = false;
};

std::mutex g_mu;
std::mutex g_aux_mu;              // one fork/join sequence on an aux stream at a time
DeviceState g_dev[kMaxDevices];

__device__ int g_status;

conv3d_status_t device_state(DeviceState*& out, int& dev) {
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device ordinal %d out of range", dev);
    return CONV3D_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.init) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&s.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                    dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    if (major != 10 || minor != 0) {
      set_error("libconv3d is built for sm_100a; device %d is sm_%d%d", dev, major, minor);
      return CONV3D_ERR_UNSUPPORTED;
    }
    void* sp = nullptr;
    if ((e = cudaGetSymbolAddress(&sp, g_status)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(status)");
    s.status = static_cast<int*>(sp);
    s.init = true;
  }
  out = &s;
  return CONV3D_OK;
}

// The device's aux stream and events, created on first use; false if they
// cannot be had (the caller then runs everything on its own stream).  They
// are not created while `caller` is being captured into a graph: that call
// runs sequentially, and a later eager call creates them.
bool aux_stream(DeviceState& s, cudaStream_t caller) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (s.aux) return true;
  if (s.aux_failed) return false;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(caller, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return false;
  }
  int least = 0, greatest = 0;
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
      cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, greatest) == cudaSuccess &&
      cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) == cudaSuccess &&
      cudaEventCreateWithFlags(&join, cudaEventDisableTiming) == cudaSuccess) {
    s.aux = st;
    s.aux_fork = fork;
    s.aux_join = join;
    return true;
  }
  if (join) cudaEventDestroy(join);
  if (fork) cudaEventDestroy(fork);
  if (st) cudaStreamDestroy(st);
  cudaGetLastError();
  s.aux_failed = true;
  return false;
}

// ------------------------------------------------------------------ tensor maps

// An activation tensor viewed as `images` images of H x W pixels with Cin
// channels; each load gathers `pixels_per_load` output pixels' windows shifted
// by one tap (the tap is the load's im2col offset).
conv3d_status_t encode_im2col(const Problem& P, const void* base, long long images,
                              int pixels_per_load, CUtensorMap& map, bool bytes8 = false) {
  // 8-bit (the e5m2 copy of x): one byte a value, 128-channel boxes
  const CUtensorMapDataType dt =
      bytes8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
             : (P.dtype == CONV3D_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  const cuuint64_t es = bytes8 ? 1 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(P.Cin), static_cast<cuuint64_t>(P.W),
                              static_cast<cuuint64_t>(P.H), static_cast<cuuint64_t>(images)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(P.Cin) * es,
                                 static_cast<cuuint64_t>(P.W) * P.Cin * es,
                                 static_cast<cuuint64_t>(P.H) * P.W * P.Cin * es};
  // Window-origin box: first origin at -pad, last at dim-1+pad-(k-1) (or, for
  // a data-gradient phase, the origin of the last of exactly Wo, Ho outputs).
  const int lower[2] = {-P.pw, -P.ph};
  const int upper[2] = {P.exact_out ? P.Wo - P.W - P.pw : P.pw - (P.kw - 1),
                        P.exact_out ? P.Ho - P.H - P.ph : P.ph - (P.kh - 1)};
  // traversal strides: consecutive output pixels' window origins are sw
  // columns (sh rows at a row wrap) apart
  const cuuint32_t estr[4] = {1, static_cast<cuuint32_t>(P.sw), static_cast<cuuint32_t>(P.sh), 1};
  CUresult r = encode_im2col_cached(&map, dt, 4, const_cast<void*>(base), dims, strides, lower, upper,
                               bytes8 ? BK8 : BK, static_cast<cuuint32_t>(pixels_per_load), estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeIm2col failed (%d)", static_cast<int>(r));
    return CONV3D_ERR_CUDA;
  }
  return CONV3D_OK;
}

conv3d_status_t encode_maps(const Problem& P, const void* x, const void* wmat, int kt_eff,
                            int b_box_rows, int pixels_per_load, CUtensorMap& map_a,
                            CUtensorMap& map_b) {
  const CUtensorMapDataType dt =
      P.dtype == CONV3D_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  conv3d_status_t st =
      encode_im2col(P, x, static_cast<long long>(P.N) * P.D, pixels_per_load, map_a);
  if (st != CONV3D_OK) return st;
  // w viewed as [Cout][taps][Cin]; a box is 64 channels of one tap for
  // b_box_rows output channels (the tile's channels, or half of them for a
  // CTA pair).
  // Channels past Cin and rows past Cout read as zero.
  {
    const int taps = kt_eff * P.kh * P.kw;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(P.Cin), static_cast<cuuint64_t>(taps),
                                static_cast<cuuint64_t>(P.Cout)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(P.Cin) * 2,
                                   static_cast<cuuint64_t>(taps) * P.Cin * 2};
    const cuuint32_t box[3] = {BK, 1, static_cast<cuuint32_t>(b_box_rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_tiled_cached(&map_b, dt, 3, const_cast<void*>(wmat), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      set_error("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
      return CONV3D_ERR_CUDA;
    }
  }
  return CONV3D_OK;
}

// The e5m2 lo weight viewed as [Cout][kh*kw][Cin] bytes; a box is 128
// channels of one spatial tap for b_box_rows output channels (128-byte rows,
// like a 64-channel box of the 16-bit weight).
conv3d_status_t encode_w8_map(const Problem& P, const void* w8, int b_box_rows, CUtensorMap& map) {
  const int taps = P.kh * P.kw;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(P.Cin), static_cast<cuuint64_t>(taps),
                              static_cast<cuuint64_t>(P.Cout)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(P.Cin),
                                 static_cast<cuuint64_t>(taps) * P.Cin};
  const cuuint32_t box[3] = {BK8, 1, static_cast<cuuint32_t>(b_box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode_tiled_cached(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(w8),
                                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled (8-bit lo weight) failed (%d)", static_cast<int>(r));
    return CONV3D_ERR_CUDA;
  }
  return CONV3D_OK;
}

// y (or the residual) viewed as [N*Do frames][Ho*Wo pixels][Cout]; a box is 32
// channels x 32 pixels of one frame, 64-byte swizzled.  Stores clip pixels
// past the frame and channels past Cout; loads read them as zero.
conv3d_status_t encode_out_map(const Problem& P, const void* base, CUtensorMap& map,
                               bool f32 = false, long long frames = -1) {
  const CUtensorMapDataType dt =
      f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
          : (P.dtype == CONV3D_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  const cuuint64_t esize = f32 ? 4 : 2;
  const cuuint64_t howo = static_cast<cuuint64_t>(P.Ho) * P.Wo;
  const cuuint64_t nframes = frames >= 0 ? static_cast<cuuint64_t>(frames)
                                          : static_cast<cuuint64_t>(P.N) * static_cast<cuuint64_t>(P.Do);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(P.Cout), howo, nframes};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(P.Cout) * esize, howo * P.Cout * esize};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode_tiled_cached(&map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE,
                              f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    return CONV3D_ERR_CUDA;
  }
  return CONV3D_OK;
}

// ------------------------------------------------------------------ launch

bool pdl_enabled() {
  static const bool on = [] {
    const char* env = getenv("CONV3D_PDL");
    return env == nullptr || env[0] != '0';
  }();
  return on;
}

// Launches `kern` (256 threads a block, no shared memory) as a programmatic
// dependent of the kernel before it on the stream, when that is enabled: its
// blocks may be scheduled before that kernel ends and wait for it in
// griddepcontrol.wait.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), int blocks, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  if (pdl_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

// Tile shape and pipeline depth for one problem.
struct LaunchPlan {
  bool pair;          // cta_group::2 over 256-row tiles (cluster of two CTAs)
  bool swap;          // transposed product: M = 128 channels, N = 256 pixels
  KernelParams kp;
  size_t smem;
  bool epi8;          // 8 epilogue warps
  size_t split_bytes; // scratch of the tail split (partials, then tickets); 0 if none
  size_t split_part_bytes;
};

// CONV3D_SPLIT (tuning and tests): 0 turns the tail split off; n in 2..8
// cuts every tile of the last round (of every round, when there is only one)
// into n pieces whatever the shape; unset: the rule in plan_launch.
int split_override() {
  const char* env = getenv("CONV3D_SPLIT");
  if (env == nullptr || env[0] == '\0') return -1;
  const int v = atoi(env);
  return v == 0 ? 0 : (v >= 2 && v <= 8 ? v : -1);
}

// split_room: bytes of scratch the tail split may use (0: no split).
conv3d_status_t plan_launch(const DeviceState& S, const Problem& P, bool bf16, size_t split_room,
                            LaunchPlan& L) {
  // The folded weight is a kt = 2 (hi, lo) kernel over the single frame; with
  // causal replicate padding both of its taps read frame 0.
  const int kt_eff = P.fold ? 2 : P.kt;
  KernelParams& kp = L.kp;
  kp = KernelParams{};
  kp.n_tiles_n = (P.Cout + 255) / 256;
  const int per_tile = (P.Cout + kp.n_tiles_n - 1) / kp.n_tiles_n;
  kp.BN = ((per_tile + 31) / 32) * 32;
  kp.co_tile = kp.BN;
  kp.D = P.fold ? 1 : P.D;
  kp.Do = P.Do;
  kp.Ho = P.Ho;
  kp.Wo = P.Wo;
  kp.H = P.H;
  kp.W = P.W;
  kp.HoWo = P.Ho * P.Wo;
  kp.Cin = P.Cin;
  kp.Cout = P.Cout;
  kp.kt = kt_eff;
  kp.kh = P.kh;
  kp.kw = P.kw;
  kp.pf = P.fold ? 1 : P.pf;
  kp.st = P.fold ? 1 : P.st;
  kp.sh = P.sh;
  kp.sw = P.sw;
  kp.ph = P.ph;
  kp.pw = P.pw;
  kp.tpad = P.fold ? 1 : static_cast<int>(P.tpad);
  kp.f32_frames = P.f32_frames;
  kp.y_frames = P.y_frames;
  kp.combine = P.combine;
  kp.gn_stats = P.gn_stats;
  kp.gn_gamma = static_cast<const uint16_t*>(P.gn_gamma);
  kp.gn_beta = static_cast<const uint16_t*>(P.gn_beta);
  kp.gn_groups = P.gn_groups;
  kp.gn_per_frame = P.gn_per_frame;
  kp.gn_silu = P.gn_silu;
  kp.gn_out = P.gn_out;
  kp.gn_out_groups = P.gn_out_groups;
  kp.y_scatter = P.y_scatter;
  kp.sc_sh = P.sc_sh;
  kp.sc_sw = P.sc_sw;
  kp.sc_rh = P.sc_rh;
  kp.sc_rw = P.sc_rw;
  kp.sc_H = P.sc_H;
  kp.sc_W = P.sc_W;
  kp.n_chunks = (P.Cin + BK - 1) / BK;
  kp.n_chunks8 = P.lo8 ? (P.Cin + BK8 - 1) / BK8 : 0;

  // A tcgen05.mma step with N < 256 takes as long as one with N = 256, so
  // layers whose channel count leaves the N side short run transposed
  // (M = 128 channels, N = 256 pixels) when that needs fewer MMA steps and
  // still gives every SM pair a tile.  A single-tap (1x1x1) layer is bound by
  // streaming x from HBM: transposed, x fills the larger operand slot (32 KB
  // of each stage instead of 16 KB), so more of it is in flight per SM; with
  // more than 8 k-blocks per tile (four epilogue warps) it runs transposed
  // whenever that needs no more steps (measured on B200 with four epilogue
  // warps: 512->256 33x128x128, 5.06 -> 5.27 TB/s; with 4 k-blocks, 256->512,
  // the transposing epilogue dominates and it lost 9%).  With at most 8
  // k-blocks the tile gets eight epilogue warps, and then the untransposed
  // variant measured as fast or faster (512->256: 159.6-159.7 against
  // 160.8-161.7 us).  CONV3D_SWAP=0/1 forces the choice.
  const long long frames_out = static_cast<long long>(P.N) * P.Do;
  const long long normal_steps = frames_out * ((kp.HoWo + BM - 1) / BM) * kp.n_tiles_n;
  const long long swap_tiles = frames_out * ((kp.HoWo + 255) / 256) * ((P.Cout + 127) / 128);
  const bool single_tap = kt_eff * P.kh * P.kw == 1 && kp.n_chunks > 8;
  L.swap = (swap_tiles < normal_steps || (single_tap && swap_tiles <= normal_steps)) &&
           swap_tiles >= S.num_sms / 2;
  if (const char* env = getenv("CONV3D_SWAP")) {
    if (env[0] == '0') L.swap = false;
    if (env[0] == '1') L.swap = true;
  }
  // CTA pairs when there is at least one wave of 256-row tiles for them (they
  // measure on par with single CTAs, so they are off unless forced);
  // CONV3D_CTA_PAIR=0/1 forces the choice (tuning and tests).
  L.pair = false;
  if (const char* env = getenv("CONV3D_CTA_PAIR")) {
    if (env[0] == '1') L.pair = true;
  }
  if (L.swap) L.pair = false;
  if (P.out_f32 || P.f32_frames > 0) L.pair = false;
  // one-CTA variants only (the fp32 epilogue exists in the single and the
  // transposed variant)
  if (P.gn_stats || P.gn_out || P.y_scatter) L.pair = false;
  if (P.lo8) L.swap = L.pair = false;   // the e5m2 lo product: one CTA, M = pixels
  if (P.combine) L.pair = false;
  const int ctas = L.pair ? 2 : 1;
  if (L.swap) {
    kp.co_tile = 128;
    kp.BN = 256;                       // N = pixels
    kp.pix_tile = 256;
    kp.n_tiles_n = (P.Cout + 127) / 128;
  } else {
    kp.pix_tile = ctas * BM;
  }
  kp.tiles_per_frame = (kp.HoWo + kp.pix_tile - 1) / kp.pix_tile;
  kp.num_tiles = P.N * P.Do * kp.tiles_per_frame * kp.n_tiles_n;
  // Tail split.  The persistent grid runs the tiles in rounds of one per SM;
  // when the last round (or the only one) is at most half full (R tiles), the
  // other SMs would idle through it.  R tiles are then cut into S pieces along
  // K (S <= SMs / R, at most 8, at least 8 k-blocks a piece); the pieces run
  // side by side on S*R SMs in the first round, and the piece that completes a
  // tile adds up the S fp32 partials (in piece order) before the usual
  // epilogue, while the whole tiles that follow keep the tensor cores busy:
  // the launch takes about T/SMs tile times instead of ceil(T/SMs).  (With the
  // pieces last, their adding-up ended the launch: measured on B200, a
  // 512-tile first frame took 129 us split in two against 124 unsplit.)  Only
  // with scratch for it (the library's own for conv3d_fwd, a region of the
  // data gradient's workspace), never for CTA pairs or strided outputs, and
  // only below 16 rounds: beyond that it saves under 1/16 of the launch, and
  // data gradients of 57 and 209 rounds (256->512 33x128x128, 128->128
  // 121x256x256) measured 3% slower with it than without.
  kp.num_items = kp.num_tiles;
  kp.split_first = kp.num_tiles;
  kp.split_s = 1;
  L.split_bytes = 0;
  L.split_part_bytes = 0;
  const int forced = split_override();
  if (split_room > 0 && forced != 0 && !L.pair && !P.y_scatter && !P.gn_stats && !P.gn_out) {
    const int U = S.num_sms;
    const int T = kp.num_tiles;
    int R = T % U;                 // the last round (all of them for a single round)
    const int kb_nominal = P.lo8 ? P.kh * P.kw * (kp.n_chunks + kp.n_chunks8)
                                 : kt_eff * P.kh * P.kw * kp.n_chunks;
    if (R == 0 && (forced > 0 || T < U)) R = T < U ? T : U;
    if (forced > 0 || (R > 0 && 2 * R <= U && T < 16 * U)) {
      int sp = forced > 0 ? forced : U / R;
      if (forced < 0) {
        if (sp > 8) sp = 8;
        while (sp > 1 && kb_nominal / sp < 8) --sp;
      }
      // no more pieces than the scratch holds
      const size_t slot = static_cast<size_t>(BM) * kp.BN * sizeof(float);
      while (sp >= 2 && static_cast<size_t>(R) * sp * slot + static_cast<size_t>(R) * 64 > split_room)
        --sp;
      if (sp >= 2) {
        kp.split_first = T - R;
        kp.split_s = sp;
        kp.num_items = T - R + R * sp;
        L.split_part_bytes = static_cast<size_t>(R) * sp * BM * kp.BN * sizeof(float);
        L.split_bytes = L.split_part_bytes + static_cast<size_t>(R) * 8 * sizeof(unsigned long long);
      }
    }
  }
  // Eight epilogue warps (two per TMEM lane quarter, each draining every
  // other 32-column chunk) where a tile has at most 8 k-blocks: there the
  // MMAs of a tile take less time than draining its 128 x 256 accumulator
  // through four warps, so the epilogue sets the pace.  Plain and split
  // launches of one CTA; CONV3D_EPI8=0/1 forces the choice where it applies.
  {
    const int kb_tile = P.lo8 ? P.kh * P.kw * (kp.n_chunks + kp.n_chunks8)
                              : kt_eff * P.kh * P.kw * kp.n_chunks;
    const bool allowed = !L.pair && !P.gn_stats && !P.gn_out && !P.y_scatter &&
                         P.f32_frames == 0 && !P.lo8 && P.combine == 0;
    L.epi8 = allowed && kb_tile <= 8;
    if (const char* env = getenv("CONV3D_EPI8")) {
      if (env[0] == '0') L.epi8 = false;
      if (env[0] == '1') L.epi8 = allowed;
    }
  }
  const int epi_mul = L.epi8 ? 2 : 1;
  const int b_stage = kp.BN / ctas * BK * 2;
  const int stage_bytes = A_STAGE_BYTES + b_stage;
  kp.has_residual = P.has_residual ? 1 : 0;
  kp.out_f32 = P.out_f32 ? 1 : 0;
  const int reserve = 1024 /*alignment slack*/ +
                      epi_mul * EPI_Y_BYTES * (kp.out_f32 || kp.f32_frames ? 2 : 1) +
                      epi_mul * EPI_Y_BYTES * (kp.has_residual ? 1 : 0) +
                      8 * (3 * MAX_STAGES + 5 + 2 * 2 * EPI_WARPS);
  int stages = (S.max_smem_optin - reserve - 64 /*static smem*/) / stage_bytes;
  if (stages > MAX_STAGES) stages = MAX_STAGES;
  if (stages < 2) {
    set_error("not enough shared memory for two pipeline stages");
    return CONV3D_ERR_UNSUPPORTED;
  }
  kp.stages = stages;
  kp.tmem_cols = pow2_at_least(2u * kp.BN);
  kp.idesc = idesc_f16(bf16, ctas * BM, kp.BN);  // swapped: M = 128 channels, N = 256 pixels
  kp.idesc8 = idesc_f8_e5m2(BM, kp.BN);
  kp.timeout_ns = kDefaultTimeoutNs;
  L.smem = static_cast<size_t>(stages) * stage_bytes + reserve;
  return CONV3D_OK;
}

template <bool kBF16, bool kPair, bool kSwap, int kFeat = 0>
conv3d_status_t launch_kernel(DeviceState& S, const LaunchPlan& L, const CUtensorMap& map_a,
                              const CUtensorMap& map_b, const CUtensorMap& map_y,
                              const CUtensorMap& map_r, const CUtensorMap& map_p,
                              const CUtensorMap& map_f, cudaStream_t stream) {
  constexpr bool kGN = (kFeat & FEAT_GN) != 0;
  auto kern = conv3d_implicit_gemm_kernel<kBF16, kPair, kSwap, kFeat>;
  const int variant = (kBF16 ? 1 : 0) + (kPair ? 2 : 0) + (kSwap ? 4 : 0) + 8 * kFeat;
  const int threads = kGN ? GN_THREADS : (kFeat & FEAT_EPI8) ? EPI8_THREADS : NUM_THREADS;
  cudaError_t e;
  int units = S.num_sms;  // co-resident CTAs (or CTA pairs)
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!S.attr_set[variant]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               S.max_smem_optin - 64);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      S.attr_set[variant] = true;
    }
    if (kPair) {
      if (S.pair_clusters <= 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (S.num_sms / 2), 1, 1);
        cfg.blockDim = dim3(threads, 1, 1);
        cfg.dynamicSmemBytes = S.max_smem_optin - 64;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (e != cudaSuccess || clusters < 1) clusters = S.num_sms / 2;
        S.pair_clusters = clusters;
      }
      units = S.pair_clusters;
    }
  }
  const int unit_count = L.kp.num_items < units ? L.kp.num_items : units;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n_attr = 0;
  if (kPair) {
    attr[n_attr].id = cudaLaunchAttributeClusterDimension;
    attr[n_attr].val.clusterDim.x = 2;
    attr[n_attr].val.clusterDim.y = 1;
    attr[n_attr].val.clusterDim.z = 1;
    ++n_attr;
  }
  // A programmatic dependent of the previous kernel on the stream: the
  // kernel's set-up overlaps that kernel's end (it waits for it before
  // touching global memory).  CONV3D_PDL=0 turns this off.
  if (pdl_enabled()) {
    attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
    ++n_attr;
  }
  cfg.gridDim = dim3((kPair ? 2 : 1) * unit_count, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n_attr;
  if (plan_log())
    fprintf(stderr,
            "libconv3d: implicit GEMM %s%s %s, %d tiles of %d pixels x %d channels, grid %d, "
            "%d k-blocks x %d taps, %d stages, %zu B shared, %s output, last %d tiles in %d "
            "pieces\n",
            kSwap ? "transposed" : kPair ? "CTA pair" : "single",
            kGN ? " with GroupNorm+SiLU of x" : (kFeat & FEAT_EPI8) ? " with 8 epilogue warps" : "",
            kBF16 ? "bf16" : "fp16",
            L.kp.num_tiles, L.kp.pix_tile, L.kp.co_tile, static_cast<int>(cfg.gridDim.x),
            L.kp.n_chunks, L.kp.kt * L.kp.kh * L.kp.kw, L.kp.stages, L.smem,
            L.kp.out_f32 ? "fp32" : L.kp.f32_frames ? "fp32 (front frames) and 16-bit" : "16-bit",
            L.kp.num_tiles - L.kp.split_first, L.kp.split_s);
  KernelParams kp = L.kp;
  kp.test_stall = take_stall(kp.timeout_ns) ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, map_a, map_b, map_y, map_r, map_p, map_f, kp);
  if (e != cudaSuccess) return cuda_fail(e, "conv3d kernel launch");
  e = launched();
  if (e != cudaSuccess) return cuda_fail(e, "conv3d kernel launch");
  return CONV3D_OK;
}

// The one-CTA instances with optional parts: the tail split, the output
// statistics, the strided output, the GroupNorm operand transform (with or
// without the statistics), the data gradient's combined front frame and its
// mixed fp32/16-bit output (each alone, split, or strided), the first frame's
// 8-bit lo product (alone or split) and the 8 epilogue warps of short-K
// launches (alone or split).  The plan never combines the split with the
// statistics, the strided output or the GroupNorm transform.
template <bool kBF16, bool kSwap>
conv3d_status_t launch_features(DeviceState& S, const LaunchPlan& L, int feat,
                                const CUtensorMap& map_a, const CUtensorMap& map_b,
                                const CUtensorMap& map_y, const CUtensorMap& map_r,
                                const CUtensorMap& map_p, const CUtensorMap& map_f,
                                cudaStream_t stream) {
  switch (feat) {
    case FEAT_SPLIT:
      return launch_kernel<kBF16, false, kSwap, FEAT_SPLIT>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_STATS:
      return launch_kernel<kBF16, false, kSwap, FEAT_STATS>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_SCATTER:
      return launch_kernel<kBF16, false, kSwap, FEAT_SCATTER>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_GN:
      return launch_kernel<kBF16, false, kSwap, FEAT_GN>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_GN | FEAT_STATS:
      return launch_kernel<kBF16, false, kSwap, FEAT_GN | FEAT_STATS>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_EPI8:
      return launch_kernel<kBF16, false, kSwap, FEAT_EPI8>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_EPI8 | FEAT_SPLIT:
      return launch_kernel<kBF16, false, kSwap, FEAT_EPI8 | FEAT_SPLIT>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_COMBINE:
      return launch_kernel<kBF16, false, kSwap, FEAT_COMBINE>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_COMBINE | FEAT_SPLIT:
      return launch_kernel<kBF16, false, kSwap, FEAT_COMBINE | FEAT_SPLIT>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_COMBINE | FEAT_SCATTER:
      return launch_kernel<kBF16, false, kSwap, FEAT_COMBINE | FEAT_SCATTER>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_MIXED:
      return launch_kernel<kBF16, false, kSwap, FEAT_MIXED>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_MIXED | FEAT_SPLIT:
      return launch_kernel<kBF16, false, kSwap, FEAT_MIXED | FEAT_SPLIT>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_MIXED | FEAT_SCATTER:
      return launch_kernel<kBF16, false, kSwap, FEAT_MIXED | FEAT_SCATTER>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    case FEAT_LO8:
      if constexpr (!kSwap)
        return launch_kernel<kBF16, false, false, FEAT_LO8>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
      break;
    case FEAT_LO8 | FEAT_SPLIT:
      if constexpr (!kSwap)
        return launch_kernel<kBF16, false, false, FEAT_LO8 | FEAT_SPLIT>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
      break;
  }
  set_error("internal: no kernel instance for feature set %d", feat);
  return CONV3D_ERR_UNSUPPORTED;
}

// Launches the main kernel with a plan from plan_launch (whose split scratch,
// if any, the caller has filled in).
conv3d_status_t launch_planned(DeviceState& S, const Problem& P, LaunchPlan& L, const void* x,
                               const void* prev, const void* wmat, const void* bias,
                               const void* residual, void* y, cudaStream_t stream) {
  const bool bf16 = P.dtype == CONV3D_BF16;
  conv3d_status_t st = CONV3D_OK;
  L.kp.bias = bias;
  L.kp.status = S.status;
  CUtensorMap map_a, map_b, map_y, map_r, map_p, map_f;
  // with the lo part in e5m2 the 16-bit weight holds the hi taps only
  const int kt_w = P.lo8 ? 1 : L.kp.kt;
  st = L.swap ? encode_maps(P, x, wmat, kt_w, L.kp.co_tile, L.kp.pix_tile, map_a, map_b)
              : encode_maps(P, x, wmat, kt_w, L.kp.BN / (L.pair ? 2 : 1), BM, map_a, map_b);
  if (st != CONV3D_OK) return st;
  if (P.f32_frames > 0) {
    // mixed output: the fp32 front frames and the 16-bit frames after them
    const long long n = P.N;
    if ((st = encode_out_map(P, y, map_y, false, n * P.y_frames)) != CONV3D_OK) return st;
    if ((st = encode_out_map(P, P.f32_out, map_f, true, n * P.f32_frames)) != CONV3D_OK)
      return st;
  } else {
    if ((st = encode_out_map(P, y, map_y, P.out_f32)) != CONV3D_OK) return st;
    map_f = map_y;  // never written: f32_frames == 0
  }
  if (residual) {
    if ((st = encode_out_map(P, residual, map_r)) != CONV3D_OK) return st;
  } else {
    map_r = map_y;  // never read: has_residual == 0
  }
  if (P.tpad == CONV3D_TPAD_CAUSAL_CACHED && P.kt > 1) {
    // the kt-1 cached frames before the chunk, read for temporal taps before frame 0
    st = encode_im2col(P, prev, static_cast<long long>(P.N) * (P.kt - 1),
                       L.swap ? L.kp.pix_tile : BM, map_p);
    if (st != CONV3D_OK) return st;
  } else {
    map_p = map_a;  // never read: no tap reads before frame 0 in this mode
  }
  if (P.lo8) {
    // the e5m2 operands of the lo product take the cached-frames and the
    // fp32-output slots, which a first frame does not use
    if ((st = encode_im2col(P, P.x8, static_cast<long long>(P.N) * P.D, BM, map_p, true)) !=
        CONV3D_OK)
      return st;
    if ((st = encode_w8_map(P, P.w8, L.kp.BN, map_f)) != CONV3D_OK) return st;
  }
  // the optional parts this launch needs (each combination is its own instance)
  int feat = 0;
  if (P.lo8) feat |= FEAT_LO8;
  if (P.f32_frames > 0) feat |= FEAT_MIXED;
  if (P.combine) feat |= FEAT_COMBINE;
  if (L.kp.split_s > 1) feat |= FEAT_SPLIT;
  if (P.gn_out) feat |= FEAT_STATS;
  if (P.y_scatter) feat |= FEAT_SCATTER;
  if (P.gn_stats) feat |= FEAT_GN;
  if (L.epi8) feat |= FEAT_EPI8;
  if (feat != 0) {   // never a CTA pair
    if (L.swap)
      return bf16 ? launch_features<true, true>(S, L, feat, map_a, map_b, map_y, map_r, map_p, map_f, stream)
                  : launch_features<false, true>(S, L, feat, map_a, map_b, map_y, map_r, map_p, map_f, stream);
    return bf16 ? launch_features<true, false>(S, L, feat, map_a, map_b, map_y, map_r, map_p, map_f, stream)
                : launch_features<false, false>(S, L, feat, map_a, map_b, map_y, map_r, map_p, map_f, stream);
  }
  if (L.swap)
    return bf16 ? launch_kernel<true, false, true>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream)
                : launch_kernel<false, false, true>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
  if (bf16)
    return L.pair ? launch_kernel<true, true, false>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream)
                  : launch_kernel<true, false, false>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
  return L.pair ? launch_kernel<false, true, false>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream)
                : launch_kernel<false, false, false>(S, L, map_a, map_b, map_y, map_r, map_p, map_f, stream);
}

// Scratch a launch may use for the tail split: `bytes` at `ptr` (256-byte
// aligned).  The tickets are cleared on the stream before the launch, so the
// region needs no state between calls.
struct SplitRegion {
  void* ptr;
  size_t bytes;
};

// Points the plan's split at `base` (partials, then tickets) with generation `gen`.
void assign_split(LaunchPlan& L, void* base, unsigned int gen) {
  char* b = static_cast<char*>(base);
  L.kp.part = reinterpret_cast<float*>(b);
  L.kp.ticket = reinterpret_cast<unsigned long long*>(b + L.split_part_bytes);
  L.kp.gen = gen;
}

// The main kernel, with a tail split only where `split` offers scratch for it.
conv3d_status_t launch_main(DeviceState& S, const Problem& P, const void* x, const void* prev,
                            const void* wmat, const void* bias, const void* residual, void* y,
                            cudaStream_t stream, const SplitRegion* split = nullptr) {
  LaunchPlan L;
  conv3d_status_t st = plan_launch(S, P, P.dtype == CONV3D_BF16, split ? split->bytes : 0, L);
  if (st != CONV3D_OK) return st;
  if (L.split_bytes > 0) {
    cudaError_t e = cudaMemsetAsync(static_cast<char*>(split->ptr) + L.split_part_bytes, 0,
                                    L.split_bytes - L.split_part_bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "split tickets clear");
    assign_split(L, split->ptr, 1u);
  }
  return launch_planned(S, P, L, x, prev, wmat, bias, residual, y, stream);
}

// conv3d_fwd's scratch for `stream` on this device, at least `need` bytes,
// zeroed when (re)allocated; also returns the next launch generation.
conv3d_status_t cached_scratch(DeviceState& S, cudaStream_t stream, size_t need, void*& ptr,
                               unsigned int& gen) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState::Scratch* sc = nullptr;
  for (int i = 0; i < S.n_scratch; ++i)
    if (S.scratch[i].stream == stream) sc = &S.scratch[i];
  if (sc == nullptr) {
    if (S.n_scratch == 16) {
      set_error("conv3d_fwd was called on more than 16 streams; use conv3d_fwd_ws");
      return CONV3D_ERR_UNSUPPORTED;
    }
    sc = &S.scratch[S.n_scratch++];
    *sc = DeviceState::Scratch{stream, nullptr, 0, 0};
  }
  if (sc->bytes < need) {
    if (sc->ptr) {
      cudaError_t e = cudaFree(sc->ptr);
      sc->ptr = nullptr;
      sc->bytes = 0;
      if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
    }
    cudaError_t e = cudaMalloc(&sc->ptr, need);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(workspace)");
    if ((e = cudaMemset(sc->ptr, 0, need)) != cudaSuccess) return cuda_fail(e, "workspace clear");
    sc->bytes = need;
  }
  if (++sc->gen == 0) ++sc->gen;
  ptr = sc->ptr;
  gen = sc->gen;
  return CONV3D_OK;
}

// folded: (first frame) ws already holds the folded (hi, lo) weight.
conv3d_status_t run(const Problem& P, const void* x, const void* w, const void* bias,
                    const void* residual, void* y, void* ws, size_t ws_bytes, bool cached_ws,
                    cudaStream_t stream, const SplitRegion* split = nullptr,
                    bool folded = false) {
  conv3d_status_t st = load_entry_points();
  if (st != CONV3D_OK) return st;
  DeviceState* S = nullptr;
  int dev = 0;
  if ((st = device_state(S, dev)) != CONV3D_OK) return st;
  const bool bf16 = P.dtype == CONV3D_BF16;
  const void* wmat = w;
  // conv3d_fwd's own scratch can also hold the e5m2 copy of x, so there the
  // first frame's lo product may run in 8 bits (CONV3D_LO8=1; Cin a multiple
  // of 16: the 8-bit tensor maps need 16-byte rows)
  Problem Q = P;
  Q.lo8 = cached_ws && P.fold && !folded && P.Cin % 16 == 0 && lo8_enabled();
  LaunchPlan L;
  const size_t room = cached_ws ? ~size_t(0) : (split ? split->bytes : 0);
  if ((st = plan_launch(*S, Q, bf16, room, L)) != CONV3D_OK) return st;
  const int kfold[3] = {P.kt, P.kh, P.kw};
  const size_t fold_need =
      !P.fold ? 0 : (Q.lo8 ? lo8_bytes(Q) : fold_bytes(P.Cin, P.Cout, kfold));   // 256-byte multiple
  if (cached_ws && fold_need + L.split_bytes > 0) {
    unsigned int gen = 0;
    if ((st = cached_scratch(*S, stream, fold_need + L.split_bytes, ws, gen)) != CONV3D_OK)
      return st;
    ws_bytes = fold_need + L.split_bytes;
    if (L.split_bytes > 0) assign_split(L, static_cast<char*>(ws) + fold_need, gen);
  } else if (L.split_bytes > 0) {   // a caller's split region (the data gradient)
    cudaError_t e = cudaMemsetAsync(static_cast<char*>(split->ptr) + L.split_part_bytes, 0,
                                    L.split_bytes - L.split_part_bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "split tickets clear");
    assign_split(L, split->ptr, 1u);
  }
  if (P.fold) {
    const size_t need = fold_need;
    if (!cached_ws) {
      if (ws == nullptr || ws_bytes < need) {
        set_error("workspace of %zu bytes required", need);
        return CONV3D_ERR_WORKSPACE;
      }
      if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        set_error("workspace must be 256-byte aligned");
        return CONV3D_ERR_ALIGNMENT;
      }
    }
    const int spatial_cin = P.kh * P.kw * P.Cin;
    const long long total = static_cast<long long>(P.Cout) * (spatial_cin / 8);   // 16-byte vectors
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > 4 * S->num_sms) blocks = 4 * S->num_sms;
    if (Q.lo8) {
      char* base = static_cast<char*>(ws);
      uint8_t* w8 = reinterpret_cast<uint8_t*>(base + lo8_hi_bytes(Q));
      uint8_t* x8 = reinterpret_cast<uint8_t*>(base + lo8_hi_bytes(Q) + lo8_w8_bytes(Q));
      const long long xn = static_cast<long long>(P.N) * P.H * P.W * P.Cin;   // one frame a sample
      long long xb = (xn / 8 + 255) / 256;
      if (xb > 8LL * S->num_sms) xb = 8LL * S->num_sms;
      if (bf16) {
        fold_taps_lo8_kernel<true><<<blocks, 256, 0, stream>>>(
            static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), w8, P.Cout, P.kt, spatial_cin);
        x_to_e5m2_kernel<true><<<static_cast<int>(xb), 256, 0, stream>>>(
            static_cast<const uint16_t*>(x), x8, xn);
      } else {
        fold_taps_lo8_kernel<false><<<blocks, 256, 0, stream>>>(
            static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), w8, P.Cout, P.kt, spatial_cin);
        x_to_e5m2_kernel<false><<<static_cast<int>(xb), 256, 0, stream>>>(
            static_cast<const uint16_t*>(x), x8, xn);
      }
      cudaError_t e = launched(2);
      if (e != cudaSuccess) return cuda_fail(e, "8-bit fold launch");
      Q.w8 = w8;
      Q.x8 = x8;
      return launch_planned(*S, Q, L, x, P.prev, ws, bias, residual, y, stream);
    }
    if (!folded) {   // (else the caller's kernel wrote it)
      if (bf16)
        fold_temporal_taps_kernel<true><<<blocks, 256, 0, stream>>>(
            static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), P.Cout, P.kt, spatial_cin);
      else
        fold_temporal_taps_kernel<false><<<blocks, 256, 0, stream>>>(
            static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), P.Cout, P.kt, spatial_cin);
      cudaError_t e = launched();
      if (e != cudaSuccess) return cuda_fail(e, "fold kernel launch");
    }
    wmat = ws;
  }
  (void)dev;
  return launch_planned(*S, P, L, x, P.prev, wmat, bias, residual, y, stream);
}

// ------------------------------------------------------------------ allocation-free entry

// Fixed scratch for conv3d_fwd_noalloc: the folded first-frame weight (hi/lo
// parts) of any problem with Cout*kh*kw*Cin <= 4,194,304.  It lives in the
// library's own device memory, so every GPU that loads the library holds these
// 16 MiB until the process exits.  In host code `g_noalloc_scratch` names a
// host-side stand-in, not a device address: the device address is looked up
// once per device with cudaGetSymbolAddress and handed to the kernels.
constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint16_t g_noalloc_scratch[kNoallocScratchBytes / 2];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set-up on first use).
conv3d_status_t noalloc_scratch(void*& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device ordinal %d out of range", dev);
    return CONV3D_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_noalloc_ptr[dev] = ptr;
  }
  out = g_noalloc_ptr[dev];
  return CONV3D_OK;
}

// ------------------------------------------------------------------ backward data pass

// dx of a stride-1 convolution is the convolution of dy with the mirrored,
// channel-transposed weight under the complementary padding ("tr").  With
// causal replicate padding frame 0 also collects the gradient of the kt-1
// copies of itself in front.  That case runs in two parts so that only frame
// 0 needs an fp32 intermediate:
//   front -- the kt frames -(kt-1)..0 of the extended gradient, in fp32 (frame
//            0's own taps included); a fold kernel sums them into dx[:, 0];
//   body  -- frames 1..D-1, straight to dx, one launch per sample (dy and dx
//            offset by one frame, so the body is the plain transposed
//            convolution of dy[n, 1:]).
// A single frame (D = 1) needs neither: dx[n, 0] = sum over taps of the 2D
// transposed convolution of dy[n, 0], i.e. the forward first-frame problem on
// dy with the transformed weight, which folds the taps into a (hi, lo) pair.
// Workspace slack for the single-frame data gradient of a strided convolution:
// each phase's folded weight starts on a 256-byte boundary (at most 64 phases).
constexpr size_t kPhaseSlack = 64 * 256;

// The data gradient's tail-split region: the partials of up to 160 pieces of a
// 128 x 256 fp32 accumulator and their tickets (160 >= the SMs of a B200, and
// the split never runs more pieces than SMs).
constexpr size_t kSplitRegionBytes =
    ((160 * (static_cast<size_t>(BM) * 256 * sizeof(float) + 64)) + 255) & ~size_t(255);

struct BwdDataPlan {
  Problem fwd;      // the forward problem being differentiated
  Problem tr;       // the whole transposed convolution (no replicate padding), or
                    // the first-frame problem (replicate padding, D = 1)
  Problem whole;    // replicate padding, D > 1, few tiles: the extended frames in fp32
                    // and frames 1.. in 16 bits, one launch (mixed output)
  bool rep;         // replicate padding, D > 1: tr with frame 0 combined, or whole + fold
  bool phased;      // spatial stride: one transposed convolution per phase
  size_t split_bytes;  // the tail-split region, after the flipped weight and ext
  size_t wt_bytes;  // flipped weight
  size_t ext_bytes; // fp32 gradient of the front frames, or the folded weight (D = 1)
};

conv3d_status_t plan_bwd_data(const void* dy, const void* w, const void* dx, int N, int Cin, int D,
                              int H, int W, int Cout, const int kernel[3], const int stride[3],
                              const int pad[3], conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                              BwdDataPlan& B) {
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED) {
    set_error("the cached-frames rule needs the cached frames: conv3d_bwd_data_cached");
    return CONV3D_ERR_UNSUPPORTED;
  }
  // validate as the forward problem x -> y (x = dx, y = dy)
  conv3d_status_t st = validate(dx, w, nullptr, nullptr, dy, N, Cin, D, H, W, Cout, kernel,
                                stride, pad, tpad, dtype, B.fwd);
  if (st != CONV3D_OK) return st;
  if (stride[0] != 1) {
    set_error("the backward data pass supports temporal stride 1 only");
    return CONV3D_ERR_UNSUPPORTED;
  }
  const Problem& F = B.fwd;
  B.phased = stride[1] != 1 || stride[2] != 1;
  if (F.pf > F.kt - 1 || F.pb > F.kt - 1 ||
      (!B.phased && (F.ph > F.kh - 1 || F.pw > F.kw - 1))) {
    set_error("the backward data pass needs pads <= kernel extent - 1");
    return CONV3D_ERR_UNSUPPORTED;
  }
  const bool rep = tpad == CONV3D_TPAD_CAUSAL_REPLICATE && F.kt > 1;
  Problem& T = B.tr;
  T = Problem{};
  T.N = N;
  T.Cin = Cout;              // dy's channels
  T.D = F.Do;
  T.H = F.Ho;
  T.W = F.Wo;
  T.Cout = Cin;              // dx's channels
  T.kt = F.kt; T.kh = F.kh; T.kw = F.kw;
  T.st = T.sh = T.sw = 1;
  T.ph = F.kh - 1 - F.ph;
  T.pw = F.kw - 1 - F.pw;
  // dx[f] gathers dy[f + it' - (kt-1-pf)]
  T.pf = F.kt - 1 - F.pf;
  T.pb = F.kt - 1 - F.pb;
  T.Do = D;
  T.Ho = H;
  T.Wo = W;
  T.tpad = CONV3D_TPAD_ZERO;  // dy frames outside [0, Do) contribute nothing
  T.dtype = dtype;
  T.has_residual = false;
  T.out_f32 = false;
  T.prev = nullptr;
  T.fold = false;
  B.rep = rep && D > 1;
  if (rep && D == 1) {
    T.tpad = CONV3D_TPAD_CAUSAL_REPLICATE;
    T.pf = F.kt - 1;
    T.pb = 0;
    T.fold = true;
  }
  if (B.rep) {
    // causal: pf = kt-1, so T.pf = 0 and output frame f reads dy[f .. f+kt-1].
    // One launch over output frames -(kt-1) .. D-1: frames -(kt-1)..0 are the
    // kt fp32 parts of dx frame 0 (frame 0's own taps in the last), frames
    // 1..D-1 go to dx in 16 bits.
    Problem& Wh = B.whole;
    Wh = T;
    Wh.pf = T.pf + F.kt - 1;
    Wh.Do = D + F.kt - 1;
    Wh.f32_frames = F.kt;
    Wh.y_frames = D;
  }
  B.wt_bytes = (static_cast<size_t>(Cout) * F.kt * F.kh * F.kw * Cin * 2 + 255) & ~size_t(255);
  B.ext_bytes = 0;
  if (B.rep)
    B.ext_bytes = (static_cast<size_t>(N) * F.kt * H * W * Cin * 4 + 255) & ~size_t(255);
  else if (T.fold)
    B.ext_bytes = ((fold_bytes(Cout, Cin, kernel) + 255) & ~size_t(255)) + kPhaseSlack;
  B.split_bytes = kSplitRegionBytes;
  return CONV3D_OK;
}

// The data gradient under causal replicate padding has two ways to give frame 0
// the gradient of its kt-1 replicated copies: its tiles run the copies' taps
// too, into the same accumulator (combined: no fp32 frames, no fold), or one
// launch writes the kt parts of frame 0 in fp32 beside the 16-bit frames and a
// fold kernel adds them (mixed).  A combined frame-0 tile carries kt(kt+1)/2
// taps against kt for the others, and the persistent grid deals tiles out in
// rounds of one per SM, so with few rounds those tiles set the launch time:
// measured on B200, 512->128 9x64x64 (144 tiles, one round) took 173 us
// combined against 131 us mixed, while with 8 or more rounds combined won
// (128->128 9x256x256: 388 against 439 us; 256->256 9x128x128: 366 against
// 376).  Combined from 4 rounds of tiles up; CONV3D_DGRAD_COMBINE=0/1 forces
// the choice.
bool combine_front(const DeviceState& S, const Problem& T) {
  const char* e = getenv("CONV3D_DGRAD_COMBINE");
  if (e != nullptr && (e[0] == '0' || e[0] == '1')) return e[0] == '1';
  Problem Cb = T;
  Cb.combine = T.kt;
  LaunchPlan L;
  if (plan_launch(S, Cb, T.dtype == CONV3D_BF16, 0, L) != CONV3D_OK) return false;
  return L.kp.num_tiles >= 4 * S.num_sms;
}

// dx[n, 0] = the rounded sum of the kt fp32 parts in ext (causal replicate padding).
conv3d_status_t fold_front(const float* ext, void* dx, int N, int D, int kt,
                           long long frame_elems, conv3d_dtype_t dtype, int sms,
                           cudaStream_t stream) {
  const long long total = static_cast<long long>(N) * (frame_elems / 8);
  int blocks = static_cast<int>((total + 255) / 256);
  if (blocks > 8 * sms) blocks = 8 * sms;
  if (dtype == CONV3D_BF16)
    fold_front_gradient_kernel<true><<<blocks, 256, 0, stream>>>(
        ext, static_cast<uint16_t*>(dx), N, D, kt, frame_elems, FoldPhase{}, 0);
  else
    fold_front_gradient_kernel<false><<<blocks, 256, 0, stream>>>(
        ext, static_cast<uint16_t*>(dx), N, D, kt, frame_elems, FoldPhase{}, 0);
  cudaError_t e = launched();
  if (e != cudaSuccess) return cuda_fail(e, "gradient fold launch");
  return CONV3D_OK;
}

// The data gradient of a convolution with spatial strides (sh, sw), temporal
// stride 1.  dx splits into sh*sw phases (rh, rw): rows h = a*sh + rh receive
// only the taps ih = qh + sh*j (qh = (rh + ph) mod sh, j < Jh), from dy rows
// a + ch - j (ch = (rh + ph - qh) / sh), i.e. phase (rh, rw) of dx is the
// stride-1 convolution of dy with the mirrored sub-kernel of those taps and
// front pads Jh-1-ch, Jw-1-cw, giving Ah x Aw outputs that the kernel's
// epilogue stores straight to their strided positions of dx.  The temporal
// direction is the stride-1 data gradient's (frame 0 combined with its
// replicated copies, or for few tiles the front frames in fp32 and a fold,
// for causal replicate padding; the first-frame fold for a single frame).
// Phases that no tap reaches (a stride larger than the kernel) are zero.
conv3d_status_t bwd_data_phases(DeviceState& S, const BwdDataPlan& B, const void* dy,
                                const void* w, void* dx, void* workspace, cudaStream_t stream,
                                const SplitRegion* split) {
  const Problem& F = B.fwd;
  const int N = F.N, Cin = F.Cin, Cout = F.Cout, D = F.D, H = F.H, W = F.W;
  const int kt = F.kt, kh = F.kh, kw = F.kw, sh = F.sh, sw = F.sw;
  const bool bf16 = F.dtype == CONV3D_BF16;
  char* wt_at = static_cast<char*>(workspace);
  char* ext_at = static_cast<char*>(workspace) + B.wt_bytes;
  conv3d_status_t st = CONV3D_OK;
  for (int rh = 0; rh < sh && rh < H; ++rh) {
    for (int rw = 0; rw < sw && rw < W; ++rw) {
      const int qh = (rh + F.ph) % sh, qw = (rw + F.pw) % sw;
      const int Jh = qh < kh ? (kh - 1 - qh) / sh + 1 : 0;
      const int Jw = qw < kw ? (kw - 1 - qw) / sw + 1 : 0;
      const int ch = (rh + F.ph - qh) / sh, cw = (rw + F.pw - qw) / sw;
      const int Ah = (H - 1 - rh) / sh + 1, Aw = (W - 1 - rw) / sw + 1;
      const FoldPhase fp{Aw, sh, sw, rh, rw, H, W, Cin};
      if (Jh == 0 || Jw == 0) {
        const long long total = static_cast<long long>(N) * D * Ah * Aw * (Cin / 8);
        int blocks = static_cast<int>((total + 255) / 256);
        if (blocks > 8 * S.num_sms) blocks = 8 * S.num_sms;
        zero_phase_kernel<<<blocks, 256, 0, stream>>>(static_cast<uint16_t*>(dx),
                                                      static_cast<long long>(N) * D, Ah, Aw, fp);
        cudaError_t e = launched();
        if (e != cudaSuccess) return cuda_fail(e, "zero phase launch");
        continue;
      }
      const int taps = kt * Jh * Jw;
      uint16_t* wt = reinterpret_cast<uint16_t*>(wt_at);
      wt_at += static_cast<size_t>(Cin) * taps * Cout * 2;   // a multiple of 16 bytes
      {
        const dim3 grid((Cin + 63) / 64, (Cout + 63) / 64, taps);
        flip_transpose_weight_kernel<<<grid, dim3(32, 8), 0, stream>>>(
            static_cast<const uint16_t*>(w), wt, Cout, taps, Cin, kh, kw, Jh, Jw, qh, qw, sh, sw);
        cudaError_t e = launched();
        if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
      }
      Problem T = B.tr;            // temporal rule and sizes of the stride-1 transposed problem
      T.kh = Jh;
      T.kw = Jw;
      T.ph = Jh - 1 - ch;
      T.pw = Jw - 1 - cw;
      T.Ho = Ah;
      T.Wo = Aw;
      T.exact_out = true;
      T.y_scatter = static_cast<uint16_t*>(dx);
      T.sc_sh = sh;
      T.sc_sw = sw;
      T.sc_rh = rh;
      T.sc_rw = rw;
      T.sc_H = H;
      T.sc_W = W;
      if (T.ph < -127 || T.ph > 127 || T.pw < -127 || T.pw > 127) {
        set_error("stride and padding out of range for the data gradient");
        return CONV3D_ERR_UNSUPPORTED;
      }
      if (T.fold) {                // one causal-replicate frame: the first-frame fold
        const int kp[3] = {kt, Jh, Jw};
        const size_t fb = fold_bytes(Cout, Cin, kp);
        st = run(T, dy, wt, nullptr, nullptr, dx, ext_at, fb, false, stream);
        ext_at += fb;              // 256-byte multiples; the workspace has the slack
        if (st != CONV3D_OK) return st;
        continue;
      }
      if (!B.rep) {
        if ((st = launch_main(S, T, dy, nullptr, wt, nullptr, nullptr, dx, stream)) != CONV3D_OK)
          return st;
        continue;
      }
      // causal replicate, D > 1: one launch, frame 0's tiles with the taps of
      // the kt-1 replicated copies before it
      if (combine_front(S, T)) {
        Problem Cb = T;
        Cb.combine = kt;
        if ((st = launch_main(S, Cb, dy, nullptr, wt, nullptr, nullptr, dx, stream, split)) !=
            CONV3D_OK)
          return st;
        continue;
      }
      // or over output frames -(kt-1)..D-1 of every sample -- the kt front
      // frames in fp32 (dense, this phase's pixels), frames 1.. straight to
      // their strided places in dx -- then the fold into frame 0
      float* ext = reinterpret_cast<float*>(ext_at);
      ext_at += static_cast<size_t>(N) * kt * Ah * Aw * Cin * 4;
      Problem Wh = T;
      Wh.pf = T.pf + kt - 1;
      Wh.Do = D + kt - 1;
      Wh.f32_frames = kt;
      Wh.y_frames = D;
      Wh.f32_out = ext;
      if ((st = launch_main(S, Wh, dy, nullptr, wt, nullptr, nullptr, dx, stream, split)) !=
          CONV3D_OK)
        return st;
      const long long frame_elems = static_cast<long long>(Ah) * Aw * Cin;
      const long long total = static_cast<long long>(N) * (frame_elems / 8);
      int blocks = static_cast<int>((total + 255) / 256);
      if (blocks > 8 * S.num_sms) blocks = 8 * S.num_sms;
      if (bf16)
        fold_front_gradient_kernel<true><<<blocks, 256, 0, stream>>>(
            ext, static_cast<uint16_t*>(dx), N, D, kt, frame_elems, fp, 1);
      else
        fold_front_gradient_kernel<false><<<blocks, 256, 0, stream>>>(
            ext, static_cast<uint16_t*>(dx), N, D, kt, frame_elems, fp, 1);
      cudaError_t e = launched();
      if (e != cudaSuccess) return cuda_fail(e, "gradient fold launch");
    }
  }
  return CONV3D_OK;
}

__global__ void selftest_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    SharedCtl ctl{&s_abort, status, timeout_ns};
    // Nothing ever arrives on `bar`: the bounded wait must give up.
    wait_bounded(smem_addr(&bar), 0, ctl, false);
  }
  __syncthreads();
}

using WgradKernel = decltype(&conv3d_wgrad_kernel<true, false, false, WG_PIX>);

// Pixels per stage: 128, or 96 where a 128-pixel stage leaves room for only
// two stages (see the launch code).  CTA pairs always fit three 128-pixel
// stages (96-pixel ones measured no faster), so they have one instance.
template <bool kBF16>
WgradKernel wgrad_kernel_of(bool swap, bool pair, int pix, bool bias, bool mix) {
  if (mix)
    return pix == 96 ? conv3d_wgrad_kernel<kBF16, true, false, 96, false, true>
                     : conv3d_wgrad_kernel<kBF16, true, false, 128, false, true>;
  if (bias)
    return pix == 96 ? conv3d_wgrad_kernel<kBF16, false, false, 96, true>
                     : conv3d_wgrad_kernel<kBF16, false, false, 128, true>;
  if (pair) return conv3d_wgrad_kernel<kBF16, false, true, 128>;
  if (swap)
    return pix == 96 ? conv3d_wgrad_kernel<kBF16, true, false, 96>
                     : conv3d_wgrad_kernel<kBF16, true, false, 128>;
  return pix == 96 ? conv3d_wgrad_kernel<kBF16, false, false, 96>
                   : conv3d_wgrad_kernel<kBF16, false, false, 128>;
}

WgradKernel wgrad_kernel_for(bool bf16, bool swap, bool pair, int pix, bool bias, bool mix) {
  return bf16 ? wgrad_kernel_of<true>(swap, pair, pix, bias, mix)
              : wgrad_kernel_of<false>(swap, pair, pix, bias, mix);
}

// Number of pixel ranges each (tap block, output-channel tile) is split into.
// The persistent grid runs units in rounds of `sms`; the cost of a choice is
// the chunks one CTA walks (rounds x chunks per unit) plus a fixed cost per
// unit for its epilogue (fp32 atomics of a 128 x BN block, about the time of
// eight 128-pixel chunks).  The cheapest split wins; ties go to fewer splits.
long long choose_wgrad_splits(long long base_units, long long total_chunks, int sms,
                              int pix_per_chunk) {
  const long long kEpilogueChunks = 8 * 128 / pix_per_chunk;
  long long best = 1;
  long long best_cost = -1;
  const long long max_splits = total_chunks < 1024 ? total_chunks : 1024;
  for (long long s = 1; s <= max_splits; ++s) {
    const long long units = base_units * s;
    const long long rounds = (units + sms - 1) / sms;
    const long long per = (total_chunks + s - 1) / s;
    const long long cost = rounds * (per + kEpilogueChunks);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
    if (rounds > 64) break;
  }
  return best;
}

}  // namespace

extern "C" {

conv3d_status_t conv3d_fwd(const void* x, const void* w, const void* bias, const void* residual,
                           void* y, int N, int Cin, int D, int H, int W, int Cout,
                           const int kernel[3], const int stride[3], const int pad[3],
                           conv3d_tpad_t tpad, conv3d_dtype_t dtype, struct CUstream_st* stream) {
  Problem P;
  conv3d_status_t st = validate(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, tpad, dtype, P);
  if (st != CONV3D_OK) return st;
  return run(P, x, w, bias, residual, y, nullptr, 0, true, stream);
}

conv3d_status_t conv3d_fwd_ws(const void* x, const void* w, const void* bias, const void* residual,
                              void* y, int N, int Cin, int D, int H, int W, int Cout,
                              const int kernel[3], const int stride[3], const int pad[3],
                              conv3d_tpad_t tpad, conv3d_dtype_t dtype, void* workspace,
                              size_t ws_bytes, struct CUstream_st* stream) {
  Problem P;
  conv3d_status_t st = validate(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, tpad, dtype, P);
  if (st != CONV3D_OK) return st;
  if (P.fold) {
    const size_t need = fold_bytes(Cin, Cout, kernel);
    if (workspace == nullptr || ws_bytes < need) {
      set_error("workspace of %zu bytes required", need);
      return CONV3D_ERR_WORKSPACE;
    }
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
      set_error("workspace must be 256-byte aligned");
      return CONV3D_ERR_ALIGNMENT;
    }
    const size_t wsz = static_cast<size_t>(Cout) * kernel[0] * kernel[1] * kernel[2] * Cin * 2;
    const size_t ysz = static_cast<size_t>(N) * P.Do * P.Ho * P.Wo * Cout * 2;
    // the main kernel reads bias and residual after the fold has written the
    // workspace, so the workspace may overlap no operand at all
    if (overlaps(workspace, need, w, wsz) || overlaps(workspace, need, y, ysz) ||
        overlaps(workspace, need, x, static_cast<size_t>(N) * D * H * W * Cin * 2) ||
        overlaps(workspace, need, residual, ysz) ||
        overlaps(workspace, need, bias, static_cast<size_t>(Cout) * 2)) {
      set_error("workspace must not overlap x, w, bias, residual or y");
      return CONV3D_ERR_INVALID_ARG;
    }
  }
  return run(P, x, w, bias, residual, y, workspace, ws_bytes, false, stream);
}

conv3d_status_t conv3d_fwd_noalloc(const void* x, const void* w, const void* bias,
                                   const void* residual, void* y, int N, int Cin, int D, int H,
                                   int W, int Cout, const int kernel[3], const int stride[3],
                                   const int pad[3], conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                   struct CUstream_st* stream) {
  Problem P;
  conv3d_status_t st = validate(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, tpad, dtype, P);
  if (st != CONV3D_OK) return st;
  if (!P.fold) return run(P, x, w, bias, residual, y, nullptr, 0, false, stream);
  const size_t need = fold_bytes(Cin, Cout, kernel);
  if (need > kNoallocScratchBytes) {
    set_error("the first-frame fold needs %zu bytes of scratch; conv3d_fwd_noalloc holds %zu "
              "(Cout*kh*kw*Cin must be <= %zu); use conv3d_fwd_ws",
              need, kNoallocScratchBytes, kNoallocScratchBytes / 4);
    return CONV3D_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((st = noalloc_scratch(scratch)) != CONV3D_OK) return st;
  return run(P, x, w, bias, residual, y, scratch, kNoallocScratchBytes, false, stream);
}

conv3d_status_t conv3d_fwd_cached(const void* x, const void* prev, const void* w,
                                  const void* bias, const void* residual, void* y, int N,
                                  int Cin, int D, int H, int W, int Cout, const int kernel[3],
                                  const int stride[3], const int pad[3], conv3d_dtype_t dtype,
                                  struct CUstream_st* stream) {
  Problem P;
  conv3d_status_t st = validate(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, CONV3D_TPAD_CAUSAL_CACHED, dtype, P, prev);
  if (st != CONV3D_OK) return st;
  return run(P, x, w, bias, residual, y, nullptr, 0, false, stream);
}

conv3d_status_t conv3d_fwd_gn(const void* x, const double* stats, const void* gamma,
                              const void* beta, int groups, int per_frame, int apply_silu,
                              const void* w, const void* bias, const void* residual, void* y,
                              int N, int Cin, int D, int H, int W, int Cout, const int kernel[3],
                              const int stride[3], const int pad[3], conv3d_tpad_t tpad,
                              conv3d_dtype_t dtype, double* out_stats, int out_groups,
                              float out_eps, struct CUstream_st* stream) {
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED) {
    set_error("the GroupNorm-fused convolution does not take cached frames");
    return CONV3D_ERR_UNSUPPORTED;
  }
  Problem P;
  conv3d_status_t st = validate(x, w, bias, residual, y, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, tpad, dtype, P);
  if (st != CONV3D_OK) return st;
  if (stats && (groups < 1 || Cin % groups != 0 || (per_frame != 0 && per_frame != 1))) {
    set_error("groups >= 1 must divide Cin and per_frame be 0 or 1");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (out_stats && (out_groups < 1 || out_groups > 64 || Cout % out_groups != 0 ||
                    !(out_eps >= 0.0f))) {
    set_error("out_groups must divide Cout and be in [1, 64], out_eps >= 0");
    return CONV3D_ERR_INVALID_ARG;
  }
  if ((stats && (reinterpret_cast<uintptr_t>(stats) & 7u)) || (stats && gamma && !aligned16(gamma)) ||
      (stats && beta && !aligned16(beta)) ||
      (out_stats && (reinterpret_cast<uintptr_t>(out_stats) & 7u))) {
    set_error("stats and out_stats must be 8-byte, gamma and beta 16-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const size_t yb = static_cast<size_t>(N) * P.Do * P.Ho * P.Wo * Cout * 2;
  const size_t sets = static_cast<size_t>(N) * (per_frame ? D : 1);
  const size_t ob = static_cast<size_t>(N) * out_groups * 16;
  if ((stats && (overlaps(y, yb, stats, sets * groups * 16) ||
                 overlaps(y, yb, gamma, Cin * 2ull) || overlaps(y, yb, beta, Cin * 2ull))) ||
      (out_stats && (overlaps(out_stats, ob, y, yb) || overlaps(out_stats, ob, x, 2ull * N * D * H * W * Cin) ||
                     (stats && overlaps(out_stats, ob, stats, sets * groups * 16))))) {
    set_error("y, stats and out_stats must not overlap each other or the inputs");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (stats) {
    P.gn_stats = stats;
    P.gn_gamma = gamma;
    P.gn_beta = beta;
    P.gn_groups = groups;
    P.gn_per_frame = per_frame;
    P.gn_silu = apply_silu ? 1 : 0;
  }
  if (out_stats) {
    cudaError_t e = cudaMemsetAsync(out_stats, 0, ob, stream);
    if (e != cudaSuccess) return cuda_fail(e, "statistics clear");
    P.gn_out = out_stats;
    P.gn_out_groups = out_groups;
  }
  if ((st = run(P, x, w, bias, residual, y, nullptr, 0, true, stream)) != CONV3D_OK) return st;
  if (out_stats) {
    const double count = static_cast<double>(P.Do) * P.Ho * P.Wo * (Cout / out_groups);
    cudaError_t e = conv3d_gn_finalize(out_stats, static_cast<long long>(N) * out_groups, count,
                                       static_cast<double>(out_eps), stream);
    if (e != cudaSuccess) return cuda_fail(e, "statistics finalize launch");
  }
  return CONV3D_OK;
}

size_t conv3d_bwd_data_workspace_bytes(int N, int Cin, int D, int H, int W, int Cout,
                                       const int kernel[3], const int pad[3], conv3d_tpad_t tpad) {
  if (!kernel || !pad || N < 1 || Cin < 1 || D < 1 || H < 1 || W < 1 || Cout < 1) return 0;
  const size_t wt = (static_cast<size_t>(Cout) * kernel[0] * kernel[1] * kernel[2] * Cin * 2 + 255) &
                    ~size_t(255);
  size_t ext = 0;
  if (tpad == CONV3D_TPAD_CAUSAL_REPLICATE && kernel[0] > 1) {
    if (D > 1)
      ext = (static_cast<size_t>(N) * kernel[0] * H * W * Cin * 4 + 255) & ~size_t(255);
    else
      ext = ((fold_bytes(Cout, Cin, kernel) + 255) & ~size_t(255)) + kPhaseSlack;
  }
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED) return wt;
  return wt + ext + kSplitRegionBytes;
}

conv3d_status_t conv3d_bwd_data(const void* dy, const void* w, void* dx, int N, int Cin, int D,
                                int H, int W, int Cout, const int kernel[3], const int stride[3],
                                const int pad[3], conv3d_tpad_t tpad, conv3d_dtype_t dtype,
                                void* workspace, size_t ws_bytes, struct CUstream_st* stream) {
  BwdDataPlan B;
  conv3d_status_t st = plan_bwd_data(dy, w, dx, N, Cin, D, H, W, Cout, kernel, stride, pad, tpad,
                                     dtype, B);
  if (st != CONV3D_OK) return st;
  const size_t need = B.wt_bytes + B.ext_bytes + B.split_bytes;
  if (workspace == nullptr || ws_bytes < need) {
    set_error("workspace of %zu bytes required", need);
    return CONV3D_ERR_WORKSPACE;
  }
  // the launches that run as one partial wave of tiles split them along K here
  const SplitRegion split{static_cast<char*>(workspace) + B.wt_bytes + B.ext_bytes, B.split_bytes};
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
    set_error("workspace must be 256-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const size_t dx_bytes = static_cast<size_t>(N) * D * H * W * Cin * 2;
  const size_t dy_bytes = static_cast<size_t>(N) * B.fwd.Do * B.fwd.Ho * B.fwd.Wo * Cout * 2;
  const size_t w_bytes = static_cast<size_t>(Cout) * kernel[0] * kernel[1] * kernel[2] * Cin * 2;
  if (overlaps(workspace, need, dx, dx_bytes) || overlaps(workspace, need, dy, dy_bytes) ||
      overlaps(workspace, need, w, w_bytes) || overlaps(dx, dx_bytes, dy, dy_bytes)) {
    set_error("dx, dy, w and the workspace must not overlap");
    return CONV3D_ERR_INVALID_ARG;
  }
  if ((st = load_entry_points()) != CONV3D_OK) return st;
  DeviceState* S = nullptr;
  int dev = 0;
  if ((st = device_state(S, dev)) != CONV3D_OK) return st;
  if (B.phased) return bwd_data_phases(*S, B, dy, w, dx, workspace, stream, &split);
  if (B.tr.fold) {
    // a single frame: mirror, transpose and fold the weight in one pass
    // straight into the first-frame path's folded-weight scratch
    void* ws = static_cast<char*>(workspace) + B.wt_bytes;
    const dim3 grid((Cin + 63) / 64, (Cout + 63) / 64, kernel[1] * kernel[2]);
    if (dtype == CONV3D_BF16)
      flip_fold_weight_kernel<true><<<grid, dim3(32, 8), 0, stream>>>(
          static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), Cout, kernel[0], kernel[1],
          kernel[2], Cin);
    else
      flip_fold_weight_kernel<false><<<grid, dim3(32, 8), 0, stream>>>(
          static_cast<const uint16_t*>(w), static_cast<uint16_t*>(ws), Cout, kernel[0], kernel[1],
          kernel[2], Cin);
    cudaError_t e = launched();
    if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
    return run(B.tr, dy, nullptr, nullptr, nullptr, dx, ws, B.ext_bytes, false, stream, &split,
               true);
  }
  uint16_t* wt = static_cast<uint16_t*>(workspace);
  {
    const int taps = kernel[0] * kernel[1] * kernel[2];
    const dim3 grid((Cin + 63) / 64, (Cout + 63) / 64, taps);
    flip_transpose_weight_kernel<<<grid, dim3(32, 8), 0, stream>>>(
        static_cast<const uint16_t*>(w), wt, Cout, taps, Cin, kernel[1], kernel[2], kernel[1],
        kernel[2], 0, 0, 1, 1);
    cudaError_t e = launched();
    if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
  }
  if (!B.rep)
    return launch_main(*S, B.tr, dy, nullptr, wt, nullptr, nullptr, dx, stream, &split);

  float* ext = reinterpret_cast<float*>(static_cast<char*>(workspace) + B.wt_bytes);
  const long long frame_elems = static_cast<long long>(H) * W * Cin;
  // One launch computes every frame: frame 0's tiles also run the taps of the
  // kt-1 virtual frames before it (the replicated copies), so frame 0 gets
  // its whole gradient in one accumulator and one rounding -- or, with few
  // rounds of tiles, frame 0's kt parts go out in fp32 and a fold adds them.
  if (combine_front(*S, B.tr)) {
    Problem Cb = B.tr;
    Cb.combine = kernel[0];
    if (plan_log())
      fprintf(stderr, "libconv3d: data gradient: %d frames x %d samples in one launch, frame 0 "
              "with its %d replicated copies\n", D, N, kernel[0] - 1);
    return launch_main(*S, Cb, dy, nullptr, wt, nullptr, nullptr, dx, stream, &split);
  }
  Problem Wh = B.whole;
  Wh.f32_out = ext;
  if (plan_log())
    fprintf(stderr, "libconv3d: data gradient: %d front frames and %d body frames x %d samples "
            "in one launch\n", kernel[0], D - 1, N);
  st = launch_main(*S, Wh, dy, nullptr, wt, nullptr, nullptr, dx, stream, &split);
  if (st != CONV3D_OK) return st;
  return fold_front(ext, dx, N, D, kernel[0], frame_elems, dtype, S->num_sms, stream);
}


size_t conv3d_bwd_weight_workspace_bytes(int Cin, int Cout, const int kernel[3]) {
  if (!kernel || Cin < 1 || Cout < 1) return 0;
  const size_t dw = static_cast<size_t>(Cout) * kernel[0] * kernel[1] * kernel[2] * Cin * 4;
  return ((dw + 255) & ~size_t(255)) + ((static_cast<size_t>(Cout) * 4 + 255) & ~size_t(255));
}

}  // extern "C"

namespace {

// dw (+ dbias) for every temporal rule; prev: the cached frames (cached mode).
conv3d_status_t bwd_weight_impl(const void* x, const void* prev, const void* dy, void* dw,
                                void* dbias, int N, int Cin, int D, int H, int W, int Cout,
                                const int kernel[3], const int stride[3], const int pad[3],
                                conv3d_tpad_t tpad, conv3d_dtype_t dtype, void* workspace,
                                size_t ws_bytes, cudaStream_t stream) {
  Problem F;
  conv3d_status_t st = validate(x, dw ? dw : workspace, nullptr, nullptr, dy, N, Cin, D, H, W,
                                Cout, kernel, stride, pad, tpad, dtype, F, prev);
  if (st != CONV3D_OK) return st;
  if (!dw) {
    set_error("dw must be non-null");
    return CONV3D_ERR_INVALID_ARG;
  }
  if (dbias && (reinterpret_cast<uintptr_t>(dbias) & 15u)) {
    set_error("dbias must be 16-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const size_t need = conv3d_bwd_weight_workspace_bytes(Cin, Cout, kernel);
  if (workspace == nullptr || ws_bytes < need) {
    set_error("workspace of %zu bytes required", need);
    return CONV3D_ERR_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
    set_error("workspace must be 256-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const long long taps = static_cast<long long>(kernel[0]) * kernel[1] * kernel[2];
  const size_t dw_elems = static_cast<size_t>(Cout) * taps * Cin;
  const size_t x_bytes = static_cast<size_t>(N) * D * H * W * Cin * 2;
  const size_t dy_bytes = static_cast<size_t>(N) * F.Do * F.Ho * F.Wo * Cout * 2;
  const size_t p_bytes = prev ? static_cast<size_t>(N) * (kernel[0] - 1) * H * W * Cin * 2 : 0;
  if (overlaps(workspace, need, x, x_bytes) || overlaps(workspace, need, dy, dy_bytes) ||
      overlaps(workspace, need, dw, dw_elems * 2) || overlaps(dw, dw_elems * 2, x, x_bytes) ||
      overlaps(dw, dw_elems * 2, dy, dy_bytes) || overlaps(workspace, need, prev, p_bytes) ||
      overlaps(dw, dw_elems * 2, prev, p_bytes)) {
    set_error("x, prev, dy, dw and the workspace must not overlap");
    return CONV3D_ERR_INVALID_ARG;
  }
  if ((st = load_entry_points()) != CONV3D_OK) return st;
  DeviceState* S = nullptr;
  int dev = 0;
  if ((st = device_state(S, dev)) != CONV3D_OK) return st;
  const bool bf16 = dtype == CONV3D_BF16;
  // A single causal-replicate frame: every temporal tap reads frame 0, so the
  // kt tap gradients are equal; the kernel computes the kt = 1 problem over
  // frame 0 and the rounding pass writes it to all kt taps.
  const bool frame0 = tpad == CONV3D_TPAD_CAUSAL_REPLICATE && D == 1 && F.kt > 1;
  const int kt_run = frame0 ? 1 : F.kt;
  const long long taps_run = static_cast<long long>(kt_run) * F.kh * F.kw;
  float* dw32 = static_cast<float*>(workspace);
  float* db32 = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         ((dw_elems * 4 + 255) & ~size_t(255)));

  WgradParams wp{};
  wp.D = F.D; wp.Do = F.Do; wp.Ho = F.Ho; wp.Wo = F.Wo; wp.HoWo = F.Ho * F.Wo;
  wp.Cin = Cin; wp.Cout = Cout;
  wp.kt = kt_run; wp.kh = F.kh; wp.kw = F.kw;
  wp.st = F.st; wp.sh = F.sh; wp.sw = F.sw;
  wp.pf = frame0 ? 0 : F.pf; wp.ph = F.ph; wp.pw = F.pw;
  wp.tpad = frame0 ? 0 : static_cast<int>(tpad);
  wp.taps = static_cast<int>(taps_run);
  wp.cblocks = (Cin + 127) / 128;
  wp.BN = Cout >= 256 ? 256 : ((Cout + 63) / 64) * 64;
  wp.co_tiles = (Cout + wp.BN - 1) / wp.BN;
  wp.c64s = Cin / 64;
  wp.ents = F.kh * F.kw * wp.c64s;
  // Entry blocks of the swapped variant: four 64-channel entries (N = 256) by
  // default; CONV3D_WGRAD_ENTRIES=3 takes three (N = 192), which leaves no
  // half-filled last block when a temporal tap has 18 entries.  Measured on
  // B200, 128->128 layers: 9x256x256 406 -> 454 us, 121x256x256 5528 -> 5900 us
  // with three: six N = 192 blocks cost more than four N = 256 and one N = 128,
  // and every block reloads the dy tile.
  wp.ent_per_block = 4;
  if (const char* env = getenv("CONV3D_WGRAD_ENTRIES"))
    if (env[0] == '3') wp.ent_per_block = 3;
  wp.eblocks = (wp.ents + wp.ent_per_block - 1) / wp.ent_per_block;
  // The swapped variant needs whole 64-channel input boxes; it wins when it
  // issues fewer MMA steps (an N = 128 step costs about as much as N = 256).
  bool swap = false;
  if (Cin % 64 == 0) {
    const long long plain_steps = taps_run * wp.cblocks * wp.co_tiles;
    const long long swap_steps = static_cast<long long>(kt_run) * wp.eblocks * ((Cout + 127) / 128);
    swap = swap_steps < plain_steps;
    if (const char* env = getenv("CONV3D_WGRAD_SWAP")) swap = env[0] == '1';
  }
  if (swap) {
    wp.BN = 128;
    wp.co_tiles = (Cout + 127) / 128;
  }
  // CTA pairs (M = 256: two 128-row blocks of one temporal tap share the dy
  // tile, each CTA loading half of it) for full 256-channel output tiles.
  // Measured on B200: +17-23% on 3x3x3 layers; a single tap (1x1x1) is
  // HBM-bound and gains nothing, so it keeps one CTA per tile.
  bool pair = !swap && wp.BN == 256 && taps_run > 1;
  if (const char* env = getenv("CONV3D_WGRAD_PAIR")) pair = pair && env[0] == '1';
  wp.pairs_per_it = (F.kh * F.kw * wp.cblocks + 1) / 2;
  const int kCtas = pair ? 2 : 1;
  int lanes = S->num_sms;   // co-resident CTAs, or CTA pairs
  // A single tap (1x1x1 and the like) is HBM-bound: its bias gradient comes
  // from one more block per output-channel tile whose A operand is a tile of
  // ones (kBias), which reads only the dy tiles that the other blocks bring
  // into L2 at the same time, instead of a second pass over dy.  It needs a
  // temporal tap whose source frame exists for every output frame, so that its
  // units walk every dy pixel; CONV3D_WGRAD_DBIAS_BLOCK=0 turns it off.
  wp.db = nullptr;
  wp.db_it = -1;
  bool bias_block = false;
  if (dbias && !swap && !pair && taps_run == 1) {
    const char* env = getenv("CONV3D_WGRAD_DBIAS_BLOCK");
    if (env == nullptr || env[0] != '0') {
      for (int it = 0; it < kt_run && wp.db_it < 0; ++it) {
        const long long f_lo = static_cast<long long>(it) - wp.pf;
        const long long f_hi = static_cast<long long>(F.Do - 1) * wp.st + it - wp.pf;
        const bool lo_ok = f_lo >= 0 || wp.tpad == 1 || wp.tpad == 3;   // replicate / cached frames
        if (lo_ok && f_hi < wp.D) wp.db_it = it;
      }
      bias_block = wp.db_it >= 0;
    }
  }
  if (bias_block) wp.db = db32;
  // Pixels per stage.  A stage holds two 64-channel x boxes and the dy boxes
  // (plain, pair) or two dy boxes and four x boxes (swapped), 128 bytes per
  // pixel each.  Three stages in flight keep the tensor cores fed; where
  // 128-pixel stages leave room for only two (six boxes: the swapped variant,
  // and one-CTA 256-channel tiles), 96-pixel stages fit three.  Measured on
  // B200: swapped 128-channel workloads 2 x 128 px 921-1113, 4 x 64 px
  // 987-1016, 3 x 96 px 1156-1260 TFLOP/s; 1x1x1 512->256 648 -> 677.
  const int boxes = swap ? 6 : 2 + wp.BN / kCtas / 64;
  // (+ 4 KB of ones, 1024-byte aligned, for the bias block)
  const int reserve = 1024 + 8 * (2 * MAX_STAGES + 5) + (bias_block ? 4096 + 1024 : 0);
  const int smem_room = S->max_smem_optin - reserve - 64;
  int pix = smem_room / (boxes * WG_PIX * 128) >= 3 ? WG_PIX : 96;
  if (const char* env = getenv("CONV3D_WGRAD_PIX")) {
    const int v = atoi(env);
    if (!pair && (v == 96 || v == 128)) pix = v;
  }
  // Swapped entry blocks numbered across the temporal taps, so that only the
  // last block of all is partly filled (with 18 entries a tap, 14 blocks of
  // four instead of 15 with three half-filled); a tap that reads zero padding
  // for a frame then loads zeros instead of skipping the chunk.
  // CONV3D_WGRAD_MIX=0 keeps the blocks within one temporal tap.
  bool mix = swap && kt_run > 1 && wp.ents % wp.ent_per_block != 0;
  if (const char* env = getenv("CONV3D_WGRAD_MIX")) mix = mix && env[0] != '0';
  auto kern = wgrad_kernel_for(bf16, swap, pair, pix, bias_block, mix);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const int kind = mix ? 4 : bias_block ? 3 : swap ? 2 : pair ? 1 : 0;
    const int wg_variant = 4 * kind + 2 * (pix == 96 ? 1 : 0) + (bf16 ? 1 : 0);
    cudaError_t e = cudaSuccess;
    if (!S->wg_attr_set[wg_variant]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               S->max_smem_optin - 64);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      S->wg_attr_set[wg_variant] = true;
    }
    if (pair) {
      if (S->wg_pair_clusters <= 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (S->num_sms / 2), 1, 1);
        cfg.blockDim = dim3(NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = S->max_smem_optin - 64;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (e != cudaSuccess || clusters < 1) clusters = S->num_sms / 2;
        S->wg_pair_clusters = clusters;
      }
      lanes = S->wg_pair_clusters;
    }
  }
  wp.chunks_per_frame = (wp.HoWo + pix - 1) / pix;
  wp.total_chunks = static_cast<long long>(N) * F.Do * wp.chunks_per_frame;
  const long long base_units =
      swap   ? (mix ? (static_cast<long long>(kt_run) * wp.ents + wp.ent_per_block - 1) / wp.ent_per_block
                    : static_cast<long long>(kt_run) * wp.eblocks) * wp.co_tiles
      : pair ? static_cast<long long>(kt_run) * wp.pairs_per_it * wp.co_tiles
             : (static_cast<long long>(wp.taps) * wp.cblocks + (bias_block ? 1 : 0)) * wp.co_tiles;
  long long splits = choose_wgrad_splits(base_units, wp.total_chunks, lanes, pix);
  if (const char* env = getenv("CONV3D_WGRAD_SPLITS")) {   // tuning: pixel ranges per unit block
    const long long v = atoll(env);
    if (v >= 1 && v <= wp.total_chunks) splits = v;
  }
  if (base_units * splits > 0x7FFFFFFFLL) {
    set_error("problem too large");
    return CONV3D_ERR_UNSUPPORTED;
  }
  wp.splits = static_cast<int>(splits);
  wp.num_units = static_cast<int>(base_units * splits);
  const int stage_bytes = boxes * pix * 128;
  int stages = smem_room / stage_bytes;
  if (stages > MAX_STAGES) stages = MAX_STAGES;
  wp.stages = stages;
  wp.acc_cols = swap ? 256u : static_cast<uint32_t>(wp.BN);
  wp.tmem_cols = pow2_at_least(2u * wp.acc_cols);
  // both operands MN-major; the swapped variant sets N per unit
  wp.idesc = idesc_f16(bf16, kCtas * BM, swap ? 256 : wp.BN) | (1u << 15) | (1u << 16);
  wp.dw = dw32;
  wp.status = S->status;
  wp.timeout_ns = kDefaultTimeoutNs;
  wp.test_stall = take_stall(wp.timeout_ns) ? 1 : 0;
  const size_t smem = static_cast<size_t>(stages) * stage_bytes + reserve;

  // x through the forward im2col map (pix pixels per load), the cached frames
  // through a second one; dy as [frames][pixels][Cout]
  CUtensorMap map_x, map_dy, map_p;
  if ((st = encode_im2col(F, x, static_cast<long long>(N) * D, pix, map_x)) != CONV3D_OK)
    return st;
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED && kernel[0] > 1) {
    if ((st = encode_im2col(F, prev, static_cast<long long>(N) * (kernel[0] - 1), pix, map_p)) !=
        CONV3D_OK)
      return st;
  } else {
    map_p = map_x;   // never read
  }
  {
    const CUtensorMapDataType dt =
        bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const cuuint64_t howo = static_cast<cuuint64_t>(F.Ho) * F.Wo;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(Cout), howo,
                                static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(F.Do)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(Cout) * 2, howo * Cout * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(pix), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_tiled_cached(&map_dy, dt, 3, const_cast<void*>(dy), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      set_error("cuTensorMapEncodeTiled (dy) failed (%d)", static_cast<int>(r));
      return CONV3D_ERR_CUDA;
    }
  }
  // Clear the fp32 sums with a kernel that lets the weight-gradient kernel
  // start at once: only that kernel's epilogue waits for the clear, so the
  // clear overlaps its first MMAs, and the rounding kernel after it is
  // launched the same way.
  // (Without programmatic launches, CONV3D_PDL=0, the clear has nothing to
  // overlap and is a plain memset.)
  cudaError_t e = cudaSuccess;
  if (!pdl_enabled()) {
    if ((e = cudaMemsetAsync(workspace, 0, need, stream)) != cudaSuccess)
      return cuda_fail(e, "workspace clear");
  } else {
    const long long n4 = static_cast<long long>(need / 16);   // a multiple of 256 bytes
    // one block per SM at most, so that a weight-gradient CTA fits beside it
    long long blocks = (n4 + 255) / 256;
    if (blocks > S->num_sms) blocks = S->num_sms;
    zero_f32x4_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<float4*>(workspace), n4);
    if ((e = launched()) != cudaSuccess) return cuda_fail(e, "workspace clear launch");
  }
  // The bias gradient reads dy once more.  Its kernel uses no shared memory,
  // so its blocks fit beside the weight-gradient CTAs, and it runs on the aux
  // stream at the same time (forked after the clear, joined before the
  // rounding); CONV3D_WGRAD_DBIAS_SIDE=0 runs it after the kernel instead.
  bool side = false;
  if (dbias && !bias_block) {
    const char* env = getenv("CONV3D_WGRAD_DBIAS_SIDE");
    side = (env == nullptr || env[0] != '0') && aux_stream(*S, stream);
  }
  std::unique_lock<std::mutex> aux_lock;
  if (side) {
    aux_lock = std::unique_lock<std::mutex>(g_aux_mu);
    e = cudaEventRecord(S->aux_fork, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(S->aux, S->aux_fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "aux stream fork");
  }
  {
    const int grid_units = wp.num_units < lanes ? wp.num_units : lanes;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    unsigned n_attr = 0;
    if (pair) {
      attr[n_attr].id = cudaLaunchAttributeClusterDimension;
      attr[n_attr].val.clusterDim.x = kCtas;
      attr[n_attr].val.clusterDim.y = 1;
      attr[n_attr].val.clusterDim.z = 1;
      ++n_attr;
    }
    if (pdl_enabled()) {   // a programmatic dependent of the clear (CONV3D_PDL=0: off)
      attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
      ++n_attr;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(kCtas * grid_units), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    if (plan_log())
      fprintf(stderr,
              "libconv3d: weight gradient %s %s, %d units (%d splits of %lld chunks of %d pixels), "
              "grid %d, %d stages, %zu B shared, bias gradient %s\n",
              swap ? (mix ? "transposed (entry blocks across taps)" : "transposed")
                   : pair ? "CTA pair" : "plain",
              bf16 ? "bf16" : "fp16",
              wp.num_units, wp.splits, wp.total_chunks, pix, static_cast<int>(cfg.gridDim.x),
              wp.stages, smem,
              bias_block ? "in the kernel (block of ones)" : dbias ? "in a pass beside it" : "none");
    e = cudaLaunchKernelEx(&cfg, kern, map_x, map_dy, map_p, wp);
    if (e != cudaSuccess) return cuda_fail(e, "wgrad kernel launch");
    launched();
  }
  {
    int blocks = static_cast<int>((dw_elems / 8 + 255) / 256);   // 8 values a thread
    if (blocks > 8 * S->num_sms) blocks = 8 * S->num_sms;
    uint16_t* d16 = static_cast<uint16_t*>(dw);
    const long long run_per_co = taps_run * Cin;
    const float* cdw = dw32;
    const float* cdb = db32;
    uint16_t* d16b = static_cast<uint16_t*>(dbias);
    const long long n_dw = static_cast<long long>(dw_elems);
    const long long n_db = dbias && bias_block ? Cout : 0;
    // a programmatic dependent of the weight-gradient kernel (it waits for it)
    if (frame0 && bf16)
      e = launch_dependent(f32_to_16_bcast_kernel<true>, blocks, stream, cdw, d16, Cout, F.kt,
                           run_per_co);
    else if (frame0)
      e = launch_dependent(f32_to_16_bcast_kernel<false>, blocks, stream, cdw, d16, Cout, F.kt,
                           run_per_co);
    else if (bf16)   // with the bias block, db is final here too: one launch for both
      e = launch_dependent(f32_to_16_kernel<true>, blocks, stream, cdw, d16, n_dw, cdb, d16b, n_db);
    else
      e = launch_dependent(f32_to_16_kernel<false>, blocks, stream, cdw, d16, n_dw, cdb, d16b, n_db);
    if (e != cudaSuccess) return cuda_fail(e, "dw conversion launch");
    if ((e = launched()) != cudaSuccess) return cuda_fail(e, "dw conversion launch");
  }
  if (dbias && !bias_block) {
    // 256-channel groups along y; about three blocks per SM in all (as many
    // as fit beside a weight-gradient CTA), the pixels split evenly between
    // the blocks of a group
    const long long pixels = static_cast<long long>(N) * F.Do * F.Ho * F.Wo;
    const int groups = (Cout + BIAS_CHANNELS - 1) / BIAS_CHANNELS;
    long long blocks = (3LL * S->num_sms + groups - 1) / groups;
    long long per = (pixels + blocks - 1) / blocks;
    if (per < 64) per = 64;
    blocks = (pixels + per - 1) / per;
    const dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(groups));
    cudaStream_t bs = side ? S->aux : stream;
    if (bf16)
      bias_grad_kernel<true><<<grid, BIAS_THREADS, 0, bs>>>(static_cast<const uint16_t*>(dy),
                                                              db32, pixels, Cout, per);
    else
      bias_grad_kernel<false><<<grid, BIAS_THREADS, 0, bs>>>(static_cast<const uint16_t*>(dy),
                                                               db32, pixels, Cout, per);
    cudaError_t le = launched();
    if (side) {
      // join even after a failed launch, so the caller's stream never runs
      // ahead of work left on the aux stream
      e = cudaEventRecord(S->aux_join, S->aux);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, S->aux_join, 0);
      aux_lock.unlock();
      if (e != cudaSuccess) return cuda_fail(e, "aux stream join");
    }
    if (le != cudaSuccess) return cuda_fail(le, "dbias launch");
  }
  if (dbias && (!bias_block || frame0)) {   // (else rounded with dw above)
    if (bf16)
      f32_to_16_kernel<true><<<1, 256, 0, stream>>>(db32, static_cast<uint16_t*>(dbias), Cout);
    else
      f32_to_16_kernel<false><<<1, 256, 0, stream>>>(db32, static_cast<uint16_t*>(dbias), Cout);
    if ((e = launched()) != cudaSuccess) return cuda_fail(e, "dbias conversion launch");
  }
  return CONV3D_OK;
}

}  // namespace

extern "C" {

conv3d_status_t conv3d_bwd_weight(const void* x, const void* dy, void* dw, void* dbias, int N,
                                  int Cin, int D, int H, int W, int Cout, const int kernel[3],
                                  const int stride[3], const int pad[3], conv3d_tpad_t tpad,
                                  conv3d_dtype_t dtype, void* workspace, size_t ws_bytes,
                                  struct CUstream_st* stream) {
  if (tpad == CONV3D_TPAD_CAUSAL_CACHED) {
    set_error("the cached-frames rule needs the cached frames: conv3d_bwd_weight_cached");
    return CONV3D_ERR_UNSUPPORTED;
  }
  return bwd_weight_impl(x, nullptr, dy, dw, dbias, N, Cin, D, H, W, Cout, kernel, stride, pad,
                         tpad, dtype, workspace, ws_bytes, stream);
}

conv3d_status_t conv3d_bwd_weight_cached(const void* x, const void* prev, const void* dy, void* dw,
                                         void* dbias, int N, int Cin, int D, int H, int W,
                                         int Cout, const int kernel[3], const int stride[3],
                                         const int pad[3], conv3d_dtype_t dtype, void* workspace,
                                         size_t ws_bytes, struct CUstream_st* stream) {
  return bwd_weight_impl(x, prev, dy, dw, dbias, N, Cin, D, H, W, Cout, kernel, stride, pad,
                         CONV3D_TPAD_CAUSAL_CACHED, dtype, workspace, ws_bytes, stream);
}

conv3d_status_t conv3d_bwd_data_cached(const void* dy, const void* w, void* dx, void* dprev, int N,
                                       int Cin, int D, int H, int W, int Cout, const int kernel[3],
                                       const int stride[3], const int pad[3], conv3d_dtype_t dtype,
                                       void* workspace, size_t ws_bytes,
                                       struct CUstream_st* stream) {
  // validate as the forward chunk problem x -> y (x = dx, prev = dprev, y = dy)
  Problem F;
  conv3d_status_t st = validate(dx, w, nullptr, nullptr, dy, N, Cin, D, H, W, Cout, kernel, stride,
                                pad, CONV3D_TPAD_CAUSAL_CACHED, dtype, F, dprev ? dprev : dx);
  if (st != CONV3D_OK) return st;
  if (stride[0] != 1 || stride[1] != 1 || stride[2] != 1) {
    set_error("the backward data pass supports stride (1,1,1) only");
    return CONV3D_ERR_UNSUPPORTED;
  }
  if (F.ph > F.kh - 1 || F.pw > F.kw - 1) {
    set_error("the backward data pass needs pads <= kernel extent - 1");
    return CONV3D_ERR_UNSUPPORTED;
  }
  const size_t need = (static_cast<size_t>(Cout) * F.kt * F.kh * F.kw * Cin * 2 + 255) & ~size_t(255);
  if (workspace == nullptr || ws_bytes < need) {
    set_error("workspace of %zu bytes required", need);
    return CONV3D_ERR_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
    set_error("workspace must be 256-byte aligned");
    return CONV3D_ERR_ALIGNMENT;
  }
  const size_t dx_bytes = static_cast<size_t>(N) * D * H * W * Cin * 2;
  const size_t dp_bytes = static_cast<size_t>(N) * (F.kt - 1) * H * W * Cin * 2;
  const size_t dy_bytes = static_cast<size_t>(N) * F.Do * F.Ho * F.Wo * Cout * 2;
  const size_t w_bytes = static_cast<size_t>(Cout) * F.kt * F.kh * F.kw * Cin * 2;
  if (overlaps(workspace, need, dx, dx_bytes) || overlaps(workspace, need, dy, dy_bytes) ||
      overlaps(workspace, need, w, w_bytes) || overlaps(dx, dx_bytes, dy, dy_bytes) ||
      overlaps(workspace, need, dprev, dp_bytes) || overlaps(dprev, dp_bytes, dy, dy_bytes) ||
      overlaps(dprev, dp_bytes, dx, dx_bytes) || overlaps(dprev, dp_bytes, w, w_bytes)) {
    set_error("dx, dprev, dy, w and the workspace must not overlap");
    return CONV3D_ERR_INVALID_ARG;
  }
  if ((st = load_entry_points()) != CONV3D_OK) return st;
  DeviceState* S = nullptr;
  int dev = 0;
  if ((st = device_state(S, dev)) != CONV3D_OK) return st;
  uint16_t* wt = static_cast<uint16_t*>(workspace);
  {
    const int taps = kernel[0] * kernel[1] * kernel[2];
    const dim3 grid((Cin + 63) / 64, (Cout + 63) / 64, taps);
    flip_transpose_weight_kernel<<<grid, dim3(32, 8), 0, stream>>>(
        static_cast<const uint16_t*>(w), wt, Cout, taps, Cin, kernel[1], kernel[2], kernel[1],
        kernel[2], 0, 0, 1, 1);
    cudaError_t e = launched();
    if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
  }
  // The chunk is the zero-padded (pt = 0) convolution of the joined clip
  // [prev; x], whose data gradient is the transposed convolution of dy: joined
  // frame e gathers dy[e + it - (kt-1)] through the mirrored weight.  Frames
  // kt-1.. of the joined clip are dx (dy frames to .. to+kt-1, pf = 0), frames
  // 0..kt-2 are dprev (pf = kt-1); one launch each, all samples at once.
  Problem T{};
  T.N = N;
  T.Cin = Cout;
  T.D = F.Do;
  T.H = F.Ho;
  T.W = F.Wo;
  T.Cout = Cin;
  T.kt = F.kt; T.kh = F.kh; T.kw = F.kw;
  T.st = T.sh = T.sw = 1;
  T.ph = F.kh - 1 - F.ph;
  T.pw = F.kw - 1 - F.pw;
  T.Ho = H;
  T.Wo = W;
  T.tpad = CONV3D_TPAD_ZERO;   // dy frames outside [0, Do) contribute nothing
  T.dtype = dtype;
  Problem Tx = T;
  Tx.pf = 0;
  Tx.pb = F.kt - 1;
  Tx.Do = D;
  st = launch_main(*S, Tx, dy, nullptr, wt, nullptr, nullptr, dx, stream);
  if (st == CONV3D_OK && dprev && F.kt > 1) {
    Problem Tp = T;
    Tp.pf = F.kt - 1;
    Tp.pb = 0;
    Tp.Do = F.kt - 1;
    st = launch_main(*S, Tp, dy, nullptr, wt, nullptr, nullptr, dprev, stream);
  }
  return st;
}

size_t conv3d_workspace_bytes(int Cin, int Cout, const int kernel[3], int D, conv3d_tpad_t tpad) {
  if (!kernel || Cin < 1 || Cout < 1 || D < 1) return 0;
  if (tpad == CONV3D_TPAD_CAUSAL_REPLICATE && D == 1 && kernel[0] > 1)
    return fold_bytes(Cin, Cout, kernel);
  return 0;
}

conv3d_status_t conv3d_output_shape(int D, int H, int W, const int kernel[3], const int stride[3],
                                    const int pad[3], conv3d_tpad_t tpad, int out_dhw[3]) {
  if (!kernel || !stride || !pad || !out_dhw || D < 1 || H < 1 || W < 1)
    return CONV3D_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (kernel[i] < 1 || stride[i] < 1 || pad[i] < 0) return CONV3D_ERR_INVALID_ARG;
  int pf, pb;
  int out[3];
  if (tpad == CONV3D_TPAD_ZERO) {
    pf = pb = pad[0];
  } else if (tpad == CONV3D_TPAD_CAUSAL_REPLICATE || tpad == CONV3D_TPAD_CAUSAL_ZERO ||
             tpad == CONV3D_TPAD_CAUSAL_CACHED) {
    pf = kernel[0] - 1;
    pb = 0;
  } else {
    return CONV3D_ERR_INVALID_ARG;
  }
  const long long ext[3] = {static_cast<long long>(D) + pf + pb, static_cast<long long>(H) + 2LL * pad[1],
                            static_cast<long long>(W) + 2LL * pad[2]};
  for (int i = 0; i < 3; ++i) {
    if (ext[i] < kernel[i]) return CONV3D_ERR_INVALID_ARG;
    out[i] = static_cast<int>((ext[i] - kernel[i]) / stride[i] + 1);
  }
  for (int i = 0; i < 3; ++i) out_dhw[i] = out[i];
  return CONV3D_OK;
}

conv3d_status_t conv3d_poll_status(struct CUstream_st* stream) {
  DeviceState* S = nullptr;
  int dev = 0;
  conv3d_status_t st = device_state(S, dev);
  if (st != CONV3D_OK) return st;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  if ((e = cudaMemcpy(&v, S->status, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "read status");
  const int zero = 0;
  if ((e = cudaMemcpy(S->status, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e, "clear status");
  return static_cast<conv3d_status_t>(v);
}

const char* conv3d_status_string(conv3d_status_t s) {
  switch (s) {
    case CONV3D_OK: return "ok";
    case CONV3D_ERR_INVALID_ARG: return "invalid argument";
    case CONV3D_ERR_UNSUPPORTED: return "unsupported problem";
    case CONV3D_ERR_ALIGNMENT: return "misaligned pointer";
    case CONV3D_ERR_CUDA: return "CUDA error";
    case CONV3D_ERR_TIMEOUT: return "device wait timed out";
    case CONV3D_ERR_DEVICE_CHECK: return "device check failed";
    case CONV3D_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* conv3d_last_error(void) { return g_last_error; }

unsigned long long conv3d_kernel_launches(void) {
  return g_kernel_launches.load(std::memory_order_relaxed);
}

void conv3d_release(void) {
  {
    std::lock_guard<std::mutex> map_lock(g_map_mu);
    g_map_cache.clear();
  }
  std::lock_guard<std::mutex> aux_lock(g_aux_mu);
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return;
  for (int d = 0; d < kMaxDevices; ++d) {
    DeviceState& s = g_dev[d];
    if (s.n_scratch > 0 || s.aux) cudaSetDevice(d);
    for (int i = 0; i < s.n_scratch; ++i)
      if (s.scratch[i].ptr) cudaFree(s.scratch[i].ptr);
    s.n_scratch = 0;
    if (s.aux) {
      // work still queued on the stream completes before its resources go
      cudaEventDestroy(s.aux_join);
      cudaEventDestroy(s.aux_fork);
      cudaStreamDestroy(s.aux);
      s.aux = nullptr;
      s.aux_fork = s.aux_join = nullptr;
    }
  }
  cudaSetDevice(cur);
}

conv3d_status_t conv3d_test_arm_stall(int launches, int timeout_ms) {
  if (launches < 0 || timeout_ms < 1 || timeout_ms > 10000) {
    set_error("launches must be >= 0 and timeout_ms in [1, 10000]");
    return CONV3D_ERR_INVALID_ARG;
  }
  g_stall_timeout_ms.store(timeout_ms);
  g_stall_launches.store(launches);
  return CONV3D_OK;
}

conv3d_status_t conv3d_selftest_wait_timeout(int timeout_ms) {
  if (timeout_ms < 1 || timeout_ms > 10000) {
    set_error("timeout_ms must be in [1, 10000]");
    return CONV3D_ERR_INVALID_ARG;
  }
  DeviceState* S = nullptr;
  int dev = 0;
  conv3d_status_t st = device_state(S, dev);
  if (st != CONV3D_OK) return st;
  cudaStream_t s;
  cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  selftest_wait_kernel<<<1, 32, 0, s>>>(S->status, static_cast<unsigned long long>(timeout_ms) * 1000000ull);
  e = launched();
  if (e != cudaSuccess) {
    cudaStreamDestroy(s);
    return cuda_fail(e, "self-test launch");
  }
  st = conv3d_poll_status(s);
  cudaStreamDestroy(s);
  return st;
}

}  // extern "C"
