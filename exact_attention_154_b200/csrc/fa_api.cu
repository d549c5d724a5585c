// fa_api.cu -- host side of libfa_sm100.so: argument checks, TMA tensor maps,
// kernel selection by head dim / dtype, persistent-grid launch on the
// caller's stream.  The C ABI is declared in include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/fa.h"
#include "fa_bwd_sm100.cuh"

namespace {

using namespace fa_sm100;

constexpr int kVersion = 1 * 10000 + 2 * 100 + 0;  // 1.2.0: local window, ALiBi, varlen
// Limit of every mbarrier wait of the kernel (2 s unless the build sets it).
#ifndef FA_WAIT_LIMIT_NS
#define FA_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr unsigned long long kWaitLimitNs = FA_WAIT_LIMIT_NS;
// Bound of every mbarrier wait of the next launches (fa_debug_set_wait_limit).
std::atomic<unsigned long long> g_wait_limit_ns{kWaitLimitNs};
constexpr int kMaxDevices = 64;

// Row-statistic scratch of fa_bwd_noalloc: a library-owned device array, one
// per device (each device's module instance has its own), so that entry point
// needs no caller workspace and allocates nothing.
constexpr long long kBwdScratchFloats = 1ll << 23;
static __device__ __align__(256) float g_bwd_scratch[kBwdScratchFloats];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// g_mutex guards only first-time set-up (the driver entry point, a device's
// attributes, a kernel's shared-memory attribute, the scratch address); the
// steady-state call path takes no lock.
std::mutex g_mutex;
std::atomic<EncodeTiledFn> g_encode{nullptr};
struct DeviceState {
  std::atomic<bool> ready{false};
  bool is_sm100 = false;
  int sm_count = 0;
  std::atomic<bool> attr_set[18] = {};
  std::atomic<bool> bwd_attr_set[8] = {};
  std::atomic<float*> bwd_scratch{nullptr};  // this device's g_bwd_scratch
};
DeviceState g_dev[kMaxDevices];

int get_encode_fn() {
  if (g_encode.load(std::memory_order_acquire)) return FA_OK;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_encode.load(std::memory_order_relaxed)) return FA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                       &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  g_encode.store(reinterpret_cast<EncodeTiledFn>(fn), std::memory_order_release);
  return FA_OK;
}

int device_state(DeviceState** out, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  DeviceState& st = g_dev[dev];
  if (!st.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!st.ready.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      st.is_sm100 = (major == 10 && minor == 0);
      st.sm_count = sms;
      st.ready.store(true, std::memory_order_release);
    }
  }
  if (!st.is_sm100) return FA_ERR_DEVICE;
  *out = &st;
  *dev_out = dev;
  return FA_OK;
}

// Sets a kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
int ensure_smem_attr(std::atomic<bool>& flag, Kernel kernel, int bytes) {
  if (flag.load(std::memory_order_acquire)) return FA_OK;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (flag.load(std::memory_order_relaxed)) return FA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  flag.store(true, std::memory_order_release);
  return FA_OK;
}

// 4-D view (d, N, H, B) of one operand with element strides (1, sn, sh, sb);
// box of 128 bytes (64 16-bit or 128 8-bit elements) x `rows` rows, 128-byte
// swizzle, zero fill.  e4m3 operands are mapped as bytes.
int encode_operand(CUtensorMap* map, const void* ptr, int dtype, int d, int N, int H, int B,
                   long long sn, long long sh, long long sb, int rows) {
  const int eb = dtype == FA_E4M3 ? 1 : 2;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)sn * eb, (cuuint64_t)sh * eb, (cuuint64_t)sb * eb};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / eb), (cuuint32_t)rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType t = dtype == FA_E4M3   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                : dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = g_encode.load(std::memory_order_acquire)(
      map, t, 4, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Tensor maps depend only on these arguments, so a thread keeps the last few
// it encoded: a repeated call on the same buffers skips the encoding.
struct MapKey {
  const void* ptr;
  long long sn, sh, sb;
  int dtype, d, N, H, B, rows;
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kMapCache = 16;
thread_local MapEntry t_maps[kMapCache];
thread_local int t_next_map = 0;

int encode_cached(CUtensorMap* map, const void* ptr, int dtype, int d, int N, int H, int B,
                  long long sn, long long sh, long long sb, int rows) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));  // padding compares equal
  key.ptr = ptr; key.sn = sn; key.sh = sh; key.sb = sb;
  key.dtype = dtype; key.d = d; key.N = N; key.H = H; key.B = B; key.rows = rows;
  for (int i = 0; i < kMapCache; ++i)
    if (t_maps[i].valid && std::memcmp(&t_maps[i].key, &key, sizeof(key)) == 0) {
      *map = t_maps[i].map;
      return FA_OK;
    }
  const int rc = encode_operand(map, ptr, dtype, d, N, H, B, sn, sh, sb, rows);
  if (rc != FA_OK) return rc;
  MapEntry& e = t_maps[t_next_map];
  t_next_map = (t_next_map + 1) % kMapCache;
  e.key = key;
  e.map = *map;
  e.valid = true;
  return FA_OK;
}

// Kernel configuration per head dim and element size: (Q tiles per work
// tile, K/V ring stages).  e4m3 tiles are half the bytes, so the ring is
// deeper; their MMAs take half the time.
template <int HD, int ELT> struct Pick;
template <int ELT> struct Pick<64, ELT> { static constexpr int QS = 2, KVS = 10; };
template <> struct Pick<128, kF16> { static constexpr int QS = 2, KVS = 4; };
template <> struct Pick<128, kBF16> { static constexpr int QS = 2, KVS = 4; };
template <> struct Pick<128, kE4M3> { static constexpr int QS = 2, KVS = 10; };
template <> struct Pick<256, kF16> { static constexpr int QS = 1, KVS = 2; };
template <> struct Pick<256, kBF16> { static constexpr int QS = 1, KVS = 2; };
template <> struct Pick<256, kE4M3> { static constexpr int QS = 1, KVS = 5; };

int q_tiles_for(int d) { return d == 256 ? 1 : 2; }

template <int HD, int ELT, bool ALIBI>
int launch(FwdParams& p, DeviceState& st, cudaStream_t stream) {
  constexpr int QS = Pick<HD, ELT>::QS, KVS = Pick<HD, ELT>::KVS;
  using C = FwdCfg<HD, QS, KVS, ELT>;
  auto kernel = fa_fwd_kernel<HD, QS, KVS, ELT, ALIBI>;
  const int slot = ((HD == 64 ? 0 : HD == 128 ? 1 : 2) * 3 + ELT) * 2 + (ALIBI ? 1 : 0);
  const int rc = ensure_smem_attr(st.attr_set[slot], kernel, C::SMEM_BYTES);
  if (rc != FA_OK) return rc;
  const int grid = p.num_tiles < st.sm_count ? p.num_tiles : st.sm_count;
  kernel<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Local window sides: -1 (unbounded) or >= 0; a side that reaches past the
// longest sequence is unbounded; with the causal mask the right side is 0.
int normalize_window(int N, int causal, int* left, int* right) {
  if (*left < -1 || *right < -1) return FA_ERR_ARG;
  if (*left >= N) *left = -1;
  if (*right >= N) *right = -1;
  if (causal) *right = 0;
  return FA_OK;
}

int check_common(int B, int H, int N, int d, float* scale, int causal, int dtype) {
  if (dtype != FA_FP16 && dtype != FA_BF16 && dtype != FA_E4M3) return FA_ERR_DTYPE;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_HEADDIM;
  if (dtype == FA_E4M3 && d == 64) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_ARG;
  if (!std::isfinite(*scale) || *scale < 0.f) return FA_ERR_ARG;
  if (*scale == 0.f) *scale = 1.0f / std::sqrt(static_cast<float>(d));
  // element counts and the tile count must fit the index types used on the device
  const long long elems = (long long)B * H * N * d;
  if (elems / d / N / H != B || elems > (1ll << 46)) return FA_ERR_ARG;
  const long long qblocks = (N + 128LL * q_tiles_for(d) - 1) / (128LL * q_tiles_for(d));
  if ((long long)B * H * qblocks > 0x7fffffffLL) return FA_ERR_ARG;
  return FA_OK;
}

// One forward problem as the kernel sees it: operand views, output layout,
// masks.  Strides are in elements.
struct Problem {
  const void *q, *k, *v;
  void* o;
  float* lse;
  int B, H, N, d;  // N: sequence length (the longest one when cu_seqlens is set)
  float scale;
  int causal, dtype;
  long long sn, sh, sb;     // q / k / v: row, head, batch
  long long osn, osh, osb;  // o
  long long lsb, lsh;       // lse: batch, head (rows are contiguous)
  int map_rows, map_batches;
  int window_left, window_right;
  const float* alibi;
  const int* cu_seqlens;
  float qk_descale, v_descale;  // e4m3: dequantisation factors; 1 otherwise
};

template <int HD, int ELT>
int launch_masks(FwdParams& p, bool alibi, DeviceState& st, cudaStream_t stream) {
  return alibi ? launch<HD, ELT, true>(p, st, stream) : launch<HD, ELT, false>(p, st, stream);
}

template <int HD>
int launch_elt(FwdParams& p, int dtype, bool alibi, DeviceState& st, cudaStream_t stream) {
  if (dtype == FA_BF16) return launch_masks<HD, kBF16>(p, alibi, st, stream);
  if (dtype == FA_FP16) return launch_masks<HD, kF16>(p, alibi, st, stream);
  if constexpr (HD >= 128) {
    // e4m3: no ALiBi variant (fa_fwd_fp8 takes none)
    if (!alibi) return launch<HD, kE4M3, false>(p, st, stream);
  }
  return FA_ERR_ARG;
}

int run(const Problem& pr, cudaStream_t stream) {
  int rc = get_encode_fn();
  if (rc != FA_OK) return rc;
  DeviceState* st = nullptr;
  int dev = 0;
  if ((rc = device_state(&st, &dev)) != FA_OK) return rc;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int R = pr.map_rows, NB = pr.map_batches;
  if ((rc = encode_cached(&p.tmap_q, pr.q, pr.dtype, pr.d, R, pr.H, NB, pr.sn, pr.sh, pr.sb,
                           128)) != FA_OK)
    return rc;
  if ((rc = encode_cached(&p.tmap_k, pr.k, pr.dtype, pr.d, R, pr.H, NB, pr.sn, pr.sh, pr.sb,
                           128)) != FA_OK)
    return rc;
  if ((rc = encode_cached(&p.tmap_v, pr.v, pr.dtype, pr.d, R, pr.H, NB, pr.sn, pr.sh, pr.sb,
                           128)) != FA_OK)
    return rc;
  if (pr.dtype != FA_E4M3 &&
      (rc = encode_cached(&p.tmap_o, pr.o, pr.dtype, pr.d, R, pr.H, NB, pr.osn, pr.osh, pr.osb,
                           128)) != FA_OK)
    return rc;
  p.o = pr.o;
  p.lse = pr.lse;
  p.o_stride_n = pr.osn;
  p.o_stride_h = pr.osh;
  p.o_stride_b = pr.osb;
  p.lse_stride_b = pr.lsb;
  p.lse_stride_h = pr.lsh;
  p.B = pr.B;
  p.H = pr.H;
  p.N = pr.N;
  p.rows_total = R;
  p.cu_seqlens = pr.cu_seqlens;
  p.causal = pr.causal;
  p.window_left = pr.window_left;
  p.window_right = pr.window_right;
  p.alibi_slopes = pr.alibi;
  p.scale_log2 = pr.scale * pr.qk_descale * 1.4426950408889634f;
  p.o_scale = pr.v_descale;
  // 2-byte outputs: strides are whole 128-byte rows (d >= 64), so the base decides
  p.o_vec32 = (reinterpret_cast<uintptr_t>(pr.o) & 31u) == 0 && (pr.osn * 2) % 32 == 0 &&
              (pr.osh * 2) % 32 == 0 && (pr.osb * 2) % 32 == 0;
  const int rows_per_tile = 128 * q_tiles_for(pr.d);
  p.num_qblocks = (pr.N + rows_per_tile - 1) / rows_per_tile;
  p.num_tiles = pr.B * pr.H * p.num_qblocks;
  p.wait_limit_ns = g_wait_limit_ns.load();

  const bool alibi = pr.alibi != nullptr;
  switch (pr.d) {
    case 64: return launch_elt<64>(p, pr.dtype, alibi, *st, stream);
    case 128: return launch_elt<128>(p, pr.dtype, alibi, *st, stream);
    default: return launch_elt<256>(p, pr.dtype, alibi, *st, stream);
  }
}

// [B, H, N, d] operands and output, [B, H, N] logsumexp.
Problem bhnd_problem(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, float scale, int causal, int dtype) {
  Problem pr;
  std::memset(&pr, 0, sizeof(pr));
  pr.q = q; pr.k = k; pr.v = v; pr.o = o; pr.lse = lse;
  pr.B = B; pr.H = H; pr.N = N; pr.d = d; pr.scale = scale; pr.causal = causal; pr.dtype = dtype;
  pr.sn = pr.osn = d;
  pr.sh = pr.osh = (long long)N * d;
  pr.sb = pr.osb = (long long)H * N * d;
  pr.lsb = (long long)H * N;
  pr.lsh = N;
  pr.map_rows = N;
  pr.map_batches = B;
  pr.window_left = pr.window_right = -1;
  pr.qk_descale = pr.v_descale = 1.f;
  return pr;
}

// qkv [B, N, 3, H, d] (q / k / v differ by H * d elements), o [B, N, H, d].
Problem packed_problem(const void* qkv, void* o, float* lse, int B, int N, int H, int d,
                       float scale, int causal, int dtype) {
  const char* base = static_cast<const char*>(qkv);
  const long long hd = (long long)H * d;
  Problem pr = bhnd_problem(base, base + 2 * hd, base + 4 * hd, o, lse, B, H, N, d, scale, causal,
                            dtype);
  pr.sn = 3 * hd;
  pr.sh = d;
  pr.sb = (long long)N * 3 * hd;
  pr.osn = hd;
  pr.osh = d;
  pr.osb = (long long)N * hd;
  return pr;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

template <int HD, bool BF16, bool KV>
int launch_bwd_kernel(const BwdParams& p, DeviceState& st, cudaStream_t stream) {
  using C = BwdCfg<HD, KV>;
  auto kernel = fa_bwd_kernel<HD, BF16, KV>;
  const int slot = (HD == 64 ? 0 : 4) + (BF16 ? 2 : 0) + (KV ? 1 : 0);
  const int rc = ensure_smem_attr(st.bwd_attr_set[slot], kernel, C::SMEM_BYTES);
  if (rc != FA_OK) return rc;
  // persistent: one CTA per SM at most, each taking units in turn
  const int grid = p.units < st.sm_count ? p.units : st.sm_count;
  kernel<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int HD, bool BF16>
int launch_bwd(const BwdParams& p, DeviceState& st, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.H * p.N;
  constexpr long long kRowsPerBlock = 256 / (HD / 8);  // bwd_dsum_kernel: HD / 8 threads a row
  bwd_dsum_kernel<HD, BF16><<<(unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, stream>>>(
      p.o, p.dout, p.dsum, rows);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  int rc = launch_bwd_kernel<HD, BF16, true>(p, st, stream);
  if (rc != FA_OK) return rc;
  return launch_bwd_kernel<HD, BF16, false>(p, st, stream);
}

}  // namespace

extern "C" {

int fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, int causal, int window_left, int window_right,
               const float* alibi_slopes, int dtype, struct CUstream_st* stream) {
  if (!q || !k || !v || !o) return FA_ERR_ARG;
  if (dtype == FA_E4M3) return FA_ERR_DTYPE;  // e4m3 goes through fa_fwd_fp8
  int rc = check_common(B, H, N, d, &scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if ((rc = normalize_window(N, causal, &window_left, &window_right)) != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned4(alibi_slopes))
    return FA_ERR_ALIGN;
  Problem pr = bhnd_problem(q, k, v, o, lse, B, H, N, d, scale, causal, dtype);
  pr.window_left = window_left;
  pr.window_right = window_right;
  pr.alibi = alibi_slopes;
  return run(pr, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, int dtype, struct CUstream_st* stream) {
  return fa_fwd_ext(q, k, v, o, lse, B, H, N, d, scale, causal, -1, -1, nullptr, dtype, stream);
}

int fa_fwd_qkvpacked_ext(const void* qkv, void* o, float* lse, int B, int N, int H, int d,
                         float scale, int causal, float dropout_p, int window_left,
                         int window_right, const float* alibi_slopes, int dtype,
                         struct CUstream_st* stream) {
  if (!qkv || !o) return FA_ERR_ARG;
  if (!(dropout_p == 0.0f)) return std::isnan(dropout_p) ? FA_ERR_ARG : FA_ERR_UNSUPPORTED;
  if (dtype == FA_E4M3) return FA_ERR_DTYPE;
  int rc = check_common(B, H, N, d, &scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if ((rc = normalize_window(N, causal, &window_left, &window_right)) != FA_OK) return rc;
  if (!aligned16(qkv) || !aligned16(o) || !aligned4(lse) || !aligned4(alibi_slopes))
    return FA_ERR_ALIGN;
  Problem pr = packed_problem(qkv, o, lse, B, N, H, d, scale, causal, dtype);
  pr.window_left = window_left;
  pr.window_right = window_right;
  pr.alibi = alibi_slopes;
  return run(pr, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_qkvpacked(const void* qkv, void* o, float* lse, int B, int N, int H, int d, float scale,
                     int causal, float dropout_p, int dtype, struct CUstream_st* stream) {
  return fa_fwd_qkvpacked_ext(qkv, o, lse, B, N, H, d, scale, causal, dropout_p, -1, -1, nullptr,
                              dtype, stream);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, float descale_q, float descale_k, float descale_v,
               int causal, struct CUstream_st* stream) {
  if (!q || !k || !v || !o) return FA_ERR_ARG;
  int rc = check_common(B, H, N, d, &scale, causal, FA_E4M3);
  if (rc != FA_OK) return rc;
  for (float f : {descale_q, descale_k, descale_v})
    if (!std::isfinite(f) || !(f > 0.f)) return FA_ERR_ARG;
  if (!std::isfinite(scale * descale_q * descale_k) || !(scale * descale_q * descale_k > 0.f))
    return FA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse))
    return FA_ERR_ALIGN;
  Problem pr = bhnd_problem(q, k, v, o, lse, B, H, N, d, scale, causal, FA_E4M3);
  pr.qk_descale = descale_q * descale_k;
  pr.v_descale = descale_v;
  if (causal) pr.window_right = 0;
  return run(pr, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens, int batch, int max_seqlen, int total, int H, int d,
                  float scale, int causal, int window_left, int window_right,
                  const float* alibi_slopes, int dtype, struct CUstream_st* stream) {
  if (!q || !k || !v || !o || !cu_seqlens) return FA_ERR_ARG;
  if (dtype == FA_E4M3) return FA_ERR_DTYPE;
  int rc = check_common(batch, H, max_seqlen, d, &scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (total < 1 || (long long)total * H * d > (1ll << 46)) return FA_ERR_ARG;
  if ((rc = normalize_window(max_seqlen, causal, &window_left, &window_right)) != FA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned4(alibi_slopes) || !aligned4(cu_seqlens))
    return FA_ERR_ALIGN;
  // q, k, v, o [total, H, d]; lse [H, total]; one tensor-map batch
  Problem pr = bhnd_problem(q, k, v, o, lse, batch, H, max_seqlen, d, scale, causal, dtype);
  pr.sn = pr.osn = (long long)H * d;
  pr.sh = pr.osh = d;
  pr.sb = pr.osb = (long long)total * H * d;
  pr.lsb = 0;
  pr.lsh = total;
  pr.map_rows = total;
  pr.map_batches = 1;
  pr.window_left = window_left;
  pr.window_right = window_right;
  pr.alibi = alibi_slopes;
  pr.cu_seqlens = cu_seqlens;
  return run(pr, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Argument checks shared by both backward entry points (workspace checked by
// the caller of this function when it has one).
int check_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
              const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
              float* scale, int causal, int dtype) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_ARG;
  int rc = check_common(B, H, N, d, scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  for (const void* t : {q, k, v, o, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if (!aligned16(t)) return FA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return FA_ERR_ALIGN;
  if ((long long)B * H * ((N + 127) / 128) > 0x7fffffffLL) return FA_ERR_ARG;
  return FA_OK;
}

// Encodes the operands and launches the three backward kernels.  A null
// `workspace` selects this device's library-owned scratch array.
int run_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
            const void* dout, void* dq, void* dk, void* dv, float* workspace, int B, int H, int N,
            int d, float scale, int causal, int dtype, cudaStream_t s) {
  int rc = get_encode_fn();
  if (rc != FA_OK) return rc;
  DeviceState* st = nullptr;
  int dev = 0;
  if ((rc = device_state(&st, &dev)) != FA_OK) return rc;
  if (workspace == nullptr) {
    float* scratch = st->bwd_scratch.load(std::memory_order_acquire);
    if (scratch == nullptr) {
      // this device's address of the array, looked up once with the device current
      std::lock_guard<std::mutex> lock(g_mutex);
      scratch = st->bwd_scratch.load(std::memory_order_relaxed);
      if (scratch == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || ptr == nullptr) {
          cudaGetLastError();
          return FA_ERR_CUDA;
        }
        scratch = static_cast<float*>(ptr);
        st->bwd_scratch.store(scratch, std::memory_order_release);
      }
    }
    workspace = scratch;
  }
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const long long sn = d, sh = (long long)N * d, sb = (long long)H * N * d;
  if ((rc = encode_cached(&p.tmap_q, q, dtype, d, N, H, B, sn, sh, sb, 128)) != FA_OK) return rc;
  if ((rc = encode_cached(&p.tmap_k, k, dtype, d, N, H, B, sn, sh, sb, 128)) != FA_OK) return rc;
  if ((rc = encode_cached(&p.tmap_v, v, dtype, d, N, H, B, sn, sh, sb, 128)) != FA_OK) return rc;
  if ((rc = encode_cached(&p.tmap_do, dout, dtype, d, N, H, B, sn, sh, sb, 128)) != FA_OK) return rc;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.dsum = workspace;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  // rows are HD 16-bit values (128 or 256 bytes), so the bases decide
  p.out_vec32 = ((reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
                  reinterpret_cast<uintptr_t>(dv)) & 31u) == 0;
  p.B = B;
  p.H = H;
  p.N = N;
  p.causal = causal;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nblk = (N + 127) / 128;
  p.units = B * H * p.nblk;
  p.wait_limit_ns = g_wait_limit_ns.load();
  const bool bf16 = dtype == FA_BF16;
  if (d == 64) return bf16 ? launch_bwd<64, true>(p, *st, s) : launch_bwd<64, false>(p, *st, s);
  return bf16 ? launch_bwd<128, true>(p, *st, s) : launch_bwd<128, false>(p, *st, s);
}

}  // namespace

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, float* workspace, int B, int H, int N,
           int d, float scale, int causal, int dtype, struct CUstream_st* stream) {
  int rc = check_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, &scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if (!workspace) return FA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0) return FA_ERR_ALIGN;
  return run_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, scale, causal, dtype,
                 reinterpret_cast<cudaStream_t>(stream));
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, int dtype, struct CUstream_st* stream) {
  int rc = check_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, &scale, causal, dtype);
  if (rc != FA_OK) return rc;
  if ((long long)B * H * N > kBwdScratchFloats) return FA_ERR_ARG;
  return run_bwd(q, k, v, o, lse, dout, dq, dk, dv, nullptr, B, H, N, d, scale, causal, dtype,
                 reinterpret_cast<cudaStream_t>(stream));
}

const char* fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_ARG: return "invalid argument";
    case FA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case FA_ERR_HEADDIM: return "head dim must be 64, 128 or 256";
    case FA_ERR_DTYPE: return "dtype must be FA_FP16 or FA_BF16";
    case FA_ERR_UNSUPPORTED: return "unsupported option (dropout_p must be 0)";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "kernel gave up on a bounded wait";
    case FA_ERR_SEQLENS: return "cu_seqlens out of range (seen by the kernel)";
    case FA_ERR_DEVICE: return "current device is not sm_100";
    default: return "unknown status";
  }
}

int fa_device_status(int clear, unsigned int* detail) {
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_fa_watchdog, sizeof(word)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_watchdog, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
  }
  if (detail) *detail = word;
  if (word == 0) return FA_OK;
  return (word >> 8) == kRoleArgs ? FA_ERR_SEQLENS : FA_ERR_TIMEOUT;
}

int fa_debug_watchdog_selftest(unsigned long long limit_ns, struct CUstream_st* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return FA_ERR_ARG;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_debug_set_wait_limit(unsigned long long limit_ns) {
  if (limit_ns != 0 && (limit_ns < 100 || limit_ns > 10000000000ull)) return FA_ERR_ARG;
  g_wait_limit_ns.store(limit_ns == 0 ? kWaitLimitNs : limit_ns);
  return FA_OK;
}

int fa_debug_exp2_poly(const float* x, float* y, int n, struct CUstream_st* stream) {
  if (!x || !y || n < 0) return FA_ERR_ARG;
  if (n == 0) return FA_OK;
  const int threads = 256, pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + threads - 1) / threads, threads, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_launch_ctas(int B, int H, int N, int d, int causal) {
  float scale = 0.f;
  int rc = check_common(B, H, N, d, &scale, causal, FA_BF16);
  if (rc != FA_OK) return rc;
  DeviceState* st = nullptr;
  int dev = 0;
  if ((rc = device_state(&st, &dev)) != FA_OK) return rc;
  const long long rows = 128LL * q_tiles_for(d);
  const long long tiles = (long long)B * H * ((N + rows - 1) / rows);
  return (int)(tiles < st->sm_count ? tiles : st->sm_count);
}

int fa_version(void) { return kVersion; }

}  // extern "C"
