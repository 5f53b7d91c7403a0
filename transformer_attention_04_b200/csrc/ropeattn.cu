// libropeattn host side: the C-ABI entry points declared in include/ropeattn.h.
// Validation, workspace, TMA descriptors and launches; every step of the attention
// itself runs in the kernels of rope.cuh, attn_fwd_sm100.cuh and decode.cuh.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/ropeattn.h"
#include "attn_fwd_sm100.cuh"
#include "decode.cuh"
#include "rope.cuh"

namespace {

__device__ unsigned int g_device_status;  // sticky kernel status (ra::kStatus*)

std::atomic<long long> g_wait_limit{1LL << 26};

// Kernel-time profiling: event pairs recorded around the main kernel of each call.
struct ProfKind {
  int device = -1;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev;
  size_t used = 0;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
bool g_prof_paused = false;  // a session's pairs are kept while calls go unrecorded
ProfKind g_prof[2];  // 0: prefill attention kernel, 1: decode split kernel

// Records the start event (returns the pair index) or -1 when profiling is off.
int prof_start(int kind, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on || g_prof_paused) return -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  ProfKind& pk = g_prof[kind];
  if (pk.device != dev) {
    if (pk.used) return -1;  // one device per profiling session
    for (auto& e : pk.ev) { cudaEventDestroy(e.first); cudaEventDestroy(e.second); }
    pk.ev.clear();
    pk.device = dev;
  }
  if (pk.used == pk.ev.size()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return -1;
    if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return -1; }
    pk.ev.emplace_back(a, b);
  }
  if (cudaEventRecord(pk.ev[pk.used].first, s) != cudaSuccess) return -1;
  return static_cast<int>(pk.used++);
}
void prof_stop(int kind, int idx, cudaStream_t s) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  cudaEventRecord(g_prof[kind].ev[idx].second, s);
}
thread_local char g_last_cuda_error[256] = "";

struct DeviceState {
  bool ready = false;
  unsigned int* status = nullptr;
  int num_sms = 0;
  bool sm100 = false;
  cudaMemPool_t pool = nullptr;  // stream-ordered pool of the call workspaces
};

// The call workspaces (rotated keys, RoPE tables, decode partials) come from a pool owned by
// the library, one per device, that keeps up to this many bytes cached across stream
// synchronisations. (The device's default pool returns its memory at every synchronisation,
// so the first call after each one would map memory again.)
constexpr unsigned long long kPoolKeepBytes = 512ull << 20;
constexpr int kMaxDevices = 64;
DeviceState g_devices[kMaxDevices];
std::mutex g_devices_mu;

ra_status cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what,
                cudaGetErrorString(e));
  return RA_ERR_CUDA;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Per-device set-up, once per device with that device current: the address of the status
// word, the SM count, the architecture check and the kernels' shared-memory limits.
ra_status device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_devices_mu);
  DeviceState& st = g_devices[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    st.sm100 = (major == 10 && minor == 0);
    st.num_sms = sms;
    if (st.sm100) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, g_device_status)) != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress(status)");
      st.status = static_cast<unsigned int*>(p);
      if ((e = set_smem(ra::attn_fwd_sm100_kernel<64>, ra::FwdCfg<64>::SMEM)) != cudaSuccess ||
          (e = set_smem(ra::attn_fwd_sm100_kernel<128>, ra::FwdCfg<128>::SMEM)) != cudaSuccess ||
          (e = set_smem(ra::decode_split_kernel<64, false>, ra::DecCfg<64>::SMEM)) != cudaSuccess ||
          (e = set_smem(ra::decode_split_kernel<128, false>, ra::DecCfg<128>::SMEM)) != cudaSuccess ||
          (e = set_smem(ra::decode_split_kernel<64, true>, ra::DecCfg<64>::SMEM)) != cudaSuccess ||
          (e = set_smem(ra::decode_split_kernel<128, true>, ra::DecCfg<128>::SMEM)) != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute");
    }
    if (st.sm100) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      if ((e = cudaMemPoolCreate(&st.pool, &props)) != cudaSuccess)
        return cuda_fail(e, "cudaMemPoolCreate");
      unsigned long long keep = kPoolKeepBytes;
      if ((e = cudaMemPoolSetAttribute(st.pool, cudaMemPoolAttrReleaseThreshold, &keep)) !=
          cudaSuccess)
        return cuda_fail(e, "cudaMemPoolSetAttribute");
    }
    st.ready = true;
  }
  if (!st.sm100) return RA_ERR_UNSUPPORTED;
  *out = &st;
  return RA_OK;
}

// cuTensorMapEncodeTiled from the driver, found once through the runtime (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over [BH, rows_alloc, D] bf16 (rows_alloc = 0: S): dims (D, S, BH), row stride D,
// slice stride rows_alloc * D elements; box (64, box_rows, 1), 128-byte swizzle; rows past S
// (and slices past BH) read as zero.
ra_status make_map(CUtensorMap* m, const void* ptr, int D, int S, long long BH, int box_rows,
                   long long rows_alloc = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "cuTensorMapEncodeTiled entry point not found");
    return RA_ERR_CUDA;
  }
  if (rows_alloc <= 0) rows_alloc = S;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(rows_alloc) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return RA_ERR_CUDA;
  }
  return RA_OK;
}

// Paged-pool maps at D = 128: dimensions (64 columns, rows, 2 column blocks, slices) with the
// column blocks 128 bytes apart, so that one box of (64, page, 2) brings a whole page: its two
// 128-byte swizzled column blocks one after the other. Half the TMA operations of two
// (64, page) boxes; the scattered 4 KB page reads are bound by that count.
ra_status make_map_dec(CUtensorMap* m, const void* ptr, int D, int S, long long BH, int box_rows,
                       long long rows_alloc = 0) {
  if (D != 128) return make_map(m, ptr, D, S, BH, box_rows, rows_alloc);
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "cuTensorMapEncodeTiled entry point not found");
    return RA_ERR_CUDA;
  }
  if (rows_alloc <= 0) rows_alloc = S;
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(S), 2, static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, 128,
                                 static_cast<cuuint64_t>(rows_alloc) * D * 2};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "cuTensorMapEncodeTiled (decode, 4-D) failed (CUresult %d)", static_cast<int>(r));
    return RA_ERR_CUDA;
  }
  return RA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Blocks of the rotation kernels: one per tile (the block scheduler balances the short blocks
// over the SMs), capped at 32 per SM for very large tensors, whose blocks then stride over
// the remaining tiles
int rot_grid(long long tiles, int num_sms) {
  return static_cast<int>(std::max<long long>(1, std::min<long long>(tiles, 32LL * num_sms)));
}

int grid_for(long long work_items, int threads, int num_sms) {
  const long long blocks = (work_items + threads - 1) / threads;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(blocks, num_sms * 16LL)));
}

constexpr float kLog2e = 1.4426950408889634f;

int decode_splits(int B, int Hkv, int G, int L, int num_sms, int requested, bool paged) {
  const int max_splits = std::max(1, (L + 63) / 64);
  if (requested > 0) return std::min(requested, max_splits);
  const long long base = static_cast<long long>(B) * Hkv * ((G + 7) / 8);
  if (!paged) {
    // Contiguous cache: the fewest splits that give every SM its two resident CTAs. Each more
    // split adds a CTA ramp per slot and a partial per head (B32 Hq64 Hkv8, 8k keys, calls
    // back to back on a B200: 1 split 164 us, 2 splits 162 us, 4 splits 168 us, 8 splits
    // 171 us).
    int s = 1;
    while (s < std::min(max_splits, 32) && base * s < 2LL * num_sms) ++s;
    return s;
  }
  // Paged pool: two decode CTAs fit on one SM, but one per SM already saturates HBM: waves
  // are counted in SMs (the same decode from 16-token pages: 2 splits 163 us, 4 splits 146 us,
  // 8 splits 152 us)
  const double slots = static_cast<double>(num_sms);
  int best = 1;
  double best_eff = -1.0;
  for (int s = 1; s <= std::min(max_splits, 32); ++s) {
    const double waves = base * s / slots;
    if (waves < 1.0 && s < max_splits && s < 32) continue;
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
    if (waves >= 2.0 && eff >= 0.95) break;
  }
  return best;
}

// Fixed device scratch of rope_attn_decode_noalloc: the per-split partials live here instead
// of in memory taken per call. Every device that loads the library holds it until exit.
constexpr size_t kDecodeScratchBytes = static_cast<size_t>(16) << 20;  // 16 MiB
__device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

// Device address of the scratch, looked up once per device with that device current (the
// array's name in host code is only a stand-in for the symbol, not a device address).
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

ra_status decode_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RA_OK;
}

// Bytes of partials for `splits` key ranges: fp32 o [B*Hq*splits*D], then (m, l) pairs.
size_t decode_partials_bytes(int B, int Hq, int D, int splits) {
  const size_t rows = static_cast<size_t>(B) * Hq * splits;
  const size_t po = (rows * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return po + rows * sizeof(float2);
}

// ------------------------------------------------------------------ RoPE table cache
// (cos, sin) of absolute positions 0 .. rows-1 for one (device, base, D), built once and kept
// for the life of the process, so that a prefill or ring block does not rebuild its table.
// A table grows to the next power of two of the positions a call needs; a grown table
// replaces the old one, which stays allocated (calls already enqueued may read it).
struct RopeTable {
  int dev;
  uint32_t base_bits;
  int D;
  long long rows;
  float2* ptr;
};
constexpr size_t kTabCacheMaxBytes = static_cast<size_t>(64) << 20;
std::mutex g_tab_mu;
std::vector<RopeTable> g_tabs;
std::vector<float2*> g_tabs_retired;

// Sets *out to a table covering positions 0 .. rows_needed-1, or to null when the call must
// build its own (too many positions, or the stream is being captured into a graph, where the
// synchronous set-up of a new table is not possible).
ra_status cached_table(const DeviceState* ds, float base, int D, long long rows_needed,
                       cudaStream_t s, const float2** out) {
  *out = nullptr;
  const size_t row_bytes = static_cast<size_t>(D / 2) * sizeof(float2);
  if (rows_needed <= 0 || static_cast<size_t>(rows_needed) * row_bytes > kTabCacheMaxBytes)
    return RA_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  uint32_t bits = 0;
  std::memcpy(&bits, &base, sizeof(bits));
  std::lock_guard<std::mutex> lock(g_tab_mu);
  RopeTable* hit = nullptr;
  for (RopeTable& t : g_tabs)
    if (t.dev == dev && t.base_bits == bits && t.D == D) hit = &t;
  if (hit && hit->rows >= rows_needed) {
    *out = hit->ptr;
    return RA_OK;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
    return RA_OK;
  long long n = 4096;
  while (n < rows_needed) n <<= 1;
  n = std::min<long long>(n, static_cast<long long>(kTabCacheMaxBytes / row_bytes));
  float2* ptr = nullptr;
  if (cudaMalloc(&ptr, static_cast<size_t>(n) * row_bytes) != cudaSuccess) {
    cudaGetLastError();  // out of memory here is not an error of the call: build per call
    return RA_OK;
  }
  ra::rope_table_kernel<<<grid_for(n * (D / 2), 256, ds->num_sms), 256, 0, s>>>(ptr, 0,
                                                                                static_cast<int>(n),
                                                                                D, base);
  // every stream may read the table once this returns
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) {
    cudaFree(ptr);
    return cuda_fail(e, "RoPE table set-up");
  }
  if (hit) {
    g_tabs_retired.push_back(hit->ptr);
    hit->ptr = ptr;
    hit->rows = n;
  } else {
    g_tabs.push_back(RopeTable{dev, bits, D, n, ptr});
  }
  *out = ptr;
  return RA_OK;
}

}  // namespace


namespace {

// ------------------------------------------------------------------ prefill
struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  void* k_cache;  // null: plain prefill over k, v
  void* v_cache;
  int S_cache;
  int B, Hq, Hkv, Sq, Sk, D;
  float rope_base;
  int pos_offset;
  int causal;
  int window;
};

// One launch of the persistent attention kernel: one CTA per SM (fewer when there are fewer
// work units), each walking its units (query tile, batch, KV group, query-head pair) of the
// longest-first order in snake order.
// A chained partial launch (p.dep_late) carries a programmatic dependency on the stream's
// previous kernel, the block before it: its CTAs start on the SMs that kernel's last wave
// leaves idle, and each waits on the device only before its first merge. Every other launch
// is plain: behind the key rotation the programmatic launch was measured slower (0.649 against
// 0.624 ms per Llama-shape call on a B200). Profiled launches are plain too, so that the
// events bracket the kernel.
ra_status launch_attn(const ra::FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                      const CUtensorMap& tv, const CUtensorMap& to, int D, int num_sms,
                      cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(std::min<long long>(p.n_units, num_sms)));
  const int pi = prof_start(0, s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(ra::kFwdThreads);
  cfg.dynamicSmemBytes = D == 64 ? ra::FwdCfg<64>::SMEM : ra::FwdCfg<128>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (p.dep_late && pi < 0) ? 1 : 0;
  cudaError_t e =
      D == 64 ? cudaLaunchKernelEx(&cfg, ra::attn_fwd_sm100_kernel<64>, tq, tk, tv, to, p)
              : cudaLaunchKernelEx(&cfg, ra::attn_fwd_sm100_kernel<128>, tq, tk, tv, to, p);
  prof_stop(0, pi, s);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "attn_fwd launch");
}

ra_status prefill_impl(const PrefillArgs& a, cudaStream_t s) {
  const int B = a.B, Hq = a.Hq, Hkv = a.Hkv, Sq = a.Sq, Sk = a.Sk, D = a.D;
  if (!a.q || !a.k || !a.v || !a.out) return RA_ERR_INVALID_ARG;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.out))
    return RA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Sk < 1 || D < 1) return RA_ERR_INVALID_ARG;
  if (Hq % Hkv) return RA_ERR_INVALID_ARG;
  if (!(a.rope_base > 0.f) || !std::isfinite(a.rope_base) || a.pos_offset < 0)
    return RA_ERR_INVALID_ARG;
  if (a.window < 0 || (a.window > 0 && !a.causal)) return RA_ERR_INVALID_ARG;
  const bool cached = a.k_cache != nullptr || a.v_cache != nullptr;
  if (cached && (!a.k_cache || !a.v_cache || !aligned16(a.k_cache) || !aligned16(a.v_cache)))
    return RA_ERR_INVALID_ARG;
  const long long T = cached ? static_cast<long long>(a.pos_offset) + Sk : Sk;  // key rows attended
  if (cached && (a.S_cache < 1 || T > a.S_cache)) return RA_ERR_INVALID_ARG;
  if (a.causal && Sq > T) return RA_ERR_INVALID_ARG;
  if (static_cast<long long>(a.pos_offset) + std::max<long long>(Sq, Sk) > 0x7fffffffLL)
    return RA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const size_t qbytes = static_cast<size_t>(B) * Hq * Sq * D * 2;
  const size_t kbytes = static_cast<size_t>(B) * Hkv * Sk * D * 2;
  if (overlap(a.out, qbytes, a.q, qbytes) || overlap(a.out, qbytes, a.k, kbytes) ||
      overlap(a.out, qbytes, a.v, kbytes))
    return RA_ERR_INVALID_ARG;
  if (cached) {
    const size_t cbytes = static_cast<size_t>(B) * Hkv * a.S_cache * D * 2;
    for (const void* c : {static_cast<const void*>(a.k_cache), static_cast<const void*>(a.v_cache)})
      if (overlap(c, cbytes, a.q, qbytes) || overlap(c, cbytes, a.k, kbytes) ||
          overlap(c, cbytes, a.v, kbytes) || overlap(c, cbytes, a.out, qbytes))
        return RA_ERR_INVALID_ARG;
    if (overlap(a.k_cache, cbytes, a.v_cache, cbytes)) return RA_ERR_INVALID_ARG;
  }
  const int G = Hq / Hkv;
  // two slots per unit: two heads of a KV group (even G) or two consecutive query tiles of
  // one head (odd G)
  const int pair_q = G % 2;
  const int n_qtiles = (Sq + 127) / 128;
  const int ppg = pair_q ? G : G / 2;
  const long long n_units =
      static_cast<long long>(pair_q ? (n_qtiles + 1) / 2 : n_qtiles) * B * Hkv * ppg;
  if (n_units > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return RA_ERR_UNSUPPORTED;

  DeviceState* ds = nullptr;
  ra_status rs = device_state(&ds);
  if (rs != RA_OK) return rs;

  // the (cos, sin) table for positions pos_offset + tab_lo .. pos_offset + Sk - 1 (covers
  // every query and new key position): from the table cache when the positions allow
  const int tab_lo = std::min(0, Sk - Sq);
  const int tab_len = Sk - tab_lo;
  const long long tab_pos0 = static_cast<long long>(a.pos_offset) + tab_lo;
  const float2* tab_cached = nullptr;
  if (tab_pos0 >= 0) {
    rs = cached_table(ds, a.rope_base, D, tab_pos0 + tab_len, s, &tab_cached);
    if (rs != RA_OK) return rs;
  }
  // workspace: rotated keys (plain prefill only), then the table when it is not cached
  const size_t krot_bytes = cached ? 0 : (kbytes + 255) & ~static_cast<size_t>(255);
  const size_t tab_bytes =
      tab_cached ? 0 : static_cast<size_t>(tab_len) * (D / 2) * sizeof(float2);
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, std::max<size_t>(krot_bytes + tab_bytes, 256),
                                          ds->pool, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync(workspace)");
  void* k_rot = ws;
  const float2* tab = tab_cached ? tab_cached + tab_pos0 * (D / 2)
                                 : reinterpret_cast<float2*>(static_cast<char*>(ws) + krot_bytes);

  // angles -> (cos, sin) table (when not cached); then K -> K' once (into the cache, with V,
  // when cached)
  if (!tab_cached)
    ra::rope_table_kernel<<<grid_for(static_cast<long long>(tab_len) * (D / 2), 256,
                                     ds->num_sms), 256, 0, s>>>(
        const_cast<float2*>(tab), tab_pos0, tab_len, D, a.rope_base);
  const long long bkv_heads = static_cast<long long>(B) * Hkv;
  if (cached)
    ra::cache_write_kernel<<<rot_grid(ra::rope_tiles(bkv_heads, Sk, D), ds->num_sms),
                             ra::kRotThreads, 0, s>>>(
        static_cast<const uint4*>(a.k), static_cast<const uint4*>(a.v),
        static_cast<uint4*>(a.k_cache), static_cast<uint4*>(a.v_cache), tab,
        static_cast<long long>(B) * Hkv, Sk, a.S_cache, a.pos_offset, D, -tab_lo);
  else
    ra::rope_rotate_kernel<true><<<rot_grid(ra::rope_tiles(bkv_heads, Sk, D), ds->num_sms),
                                   ra::kRotThreads, 0, s>>>(
        static_cast<const uint4*>(a.k), static_cast<uint4*>(k_rot), tab, bkv_heads * Sk, Sk, D, 0,
        -tab_lo, a.rope_base, Sk, Sk);

  CUtensorMap tq, tk, tv, to;
  const long long bkv = static_cast<long long>(B) * Hkv;
  rs = make_map(&tq, a.q, D, Sq, static_cast<long long>(B) * Hq, 128);
  // the output tiles leave through shared memory with TMA, in Q's geometry
  if (rs == RA_OK) rs = make_map(&to, a.out, D, Sq, static_cast<long long>(B) * Hq, 128);
  if (rs == RA_OK)
    rs = cached ? make_map(&tk, a.k_cache, D, static_cast<int>(T), bkv, 128, a.S_cache)
                : make_map(&tk, k_rot, D, Sk, bkv, 128);
  if (rs == RA_OK)
    rs = cached ? make_map(&tv, a.v_cache, D, static_cast<int>(T), bkv, 128, a.S_cache)
                : make_map(&tv, a.v, D, Sk, bkv, 128);
  if (rs == RA_OK) {
    ra::FwdParams p;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.tab = tab;
    p.status = ds->status;
    p.wait_limit = g_wait_limit.load();
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Sk = static_cast<int>(T);
    p.G = G;
    p.n_slots = 2;
    p.pair_q = pair_q;
    p.ppg = ppg;
    p.n_qtiles = n_qtiles;
    p.n_units = static_cast<int>(n_units);
    p.causal = a.causal ? 1 : 0;
    p.off = static_cast<int>(T) - Sq;  // bottom-right alignment of the queries on the keys
    p.off2 = p.off;
    p.window = a.window;
    p.q_tab_off = (Sk - Sq) - tab_lo;
    p.q_split = Sq;
    p.q_tab_off2 = p.q_tab_off;
    p.scale_log2 = kLog2e / std::sqrt(static_cast<float>(D));
    p.rope_base = a.rope_base;
    p.o_acc = nullptr;
    p.lse_acc = nullptr;
    p.accumulate = 0;
    p.acc_rows = Sq;
    p.dep_late = 0;
    rs = launch_attn(p, tq, tk, tv, to, D, ds->num_sms, s);
  }
  cudaError_t ef = cudaFreeAsync(ws, s);
  if (rs == RA_OK && ef != cudaSuccess) rs = cuda_fail(ef, "cudaFreeAsync(workspace)");
  return rs;
}

// ------------------------------------------------------------------ ring attention block
struct PartialArgs {
  const void* q;
  const void* k_rot;
  const void* v;
  float* o_acc;
  float* lse_acc;
  void* out;  // optional bf16 copy of the merged result
  int B, Hq, Hkv, Sq, Sk, D;
  float rope_base;
  int q_pos0, k_pos0;
  int causal;
  int accumulate;
  int q_rows, kv_rows, acc_rows;  // rows between consecutive heads (0: packed)
  int q_split, q_pos1;            // rows >= q_split sit at q_pos1 + (i - q_split)
};

ra_status partial_impl(const PartialArgs& a, cudaStream_t s) {
  const int B = a.B, Hq = a.Hq, Hkv = a.Hkv, Sq = a.Sq, Sk = a.Sk, D = a.D;
  if (a.q_rows < 0 || a.kv_rows < 0 || a.acc_rows < 0) return RA_ERR_INVALID_ARG;
  const int q_rows = a.q_rows ? a.q_rows : Sq;
  const int kv_rows = a.kv_rows ? a.kv_rows : Sk;
  const int acc_rows = a.acc_rows ? a.acc_rows : Sq;
  if (q_rows < Sq || kv_rows < Sk || acc_rows < Sq) return RA_ERR_INVALID_ARG;
  // a second query segment (rows q_split.. at q_pos1..): under the mask every row of it must
  // see the block's first key, and q_split must fall on a work unit's edge (checked below)
  const bool two_seg = a.q_split > 0 && a.q_split < Sq;
  if (a.q_split < 0 || (two_seg && (a.q_pos1 < 0 || (a.causal && a.q_pos1 < a.k_pos0) ||
                                    static_cast<long long>(a.q_pos1) + (Sq - a.q_split) >
                                        (1LL << 30))))
    return RA_ERR_INVALID_ARG;
  if (!a.q || !a.k_rot || !a.v || !a.o_acc || !a.lse_acc) return RA_ERR_INVALID_ARG;
  if (!aligned16(a.q) || !aligned16(a.k_rot) || !aligned16(a.v) || !aligned16(a.o_acc) ||
      (reinterpret_cast<uintptr_t>(a.lse_acc) & 3u) || (a.out && !aligned16(a.out)))
    return RA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Sk < 1 || D < 1) return RA_ERR_INVALID_ARG;
  if (Hq % Hkv) return RA_ERR_INVALID_ARG;
  if (!(a.rope_base > 0.f) || !std::isfinite(a.rope_base)) return RA_ERR_INVALID_ARG;
  // positions stay below 2^30 so that every row and key index sum fits an int
  if (a.q_pos0 < 0 || a.k_pos0 < 0 || static_cast<long long>(a.q_pos0) + Sq > (1LL << 30) ||
      static_cast<long long>(a.k_pos0) + Sk > (1LL << 30))
    return RA_ERR_INVALID_ARG;
  // under the causal mask every query row must see the block's first key
  if (a.causal && a.q_pos0 < a.k_pos0) return RA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  // extents of the strided views: (heads - 1) full strides plus the last head's rows
  auto extent = [](long long heads, long long rows, long long used, long long row_bytes) {
    return static_cast<size_t>(((heads - 1) * rows + used) * row_bytes);
  };
  const long long bhq = static_cast<long long>(B) * Hq, bhk = static_cast<long long>(B) * Hkv;
  const size_t qbytes = extent(bhq, q_rows, Sq, 2LL * D);
  const size_t kbytes = extent(bhk, kv_rows, Sk, 2LL * D);
  const size_t obytes = extent(bhq, acc_rows, Sq, 4LL * D);
  const size_t lbytes = extent(bhq, acc_rows, Sq, 4);
  const size_t outbytes = extent(bhq, acc_rows, Sq, 2LL * D);
  for (const auto& w : {std::make_pair(static_cast<const void*>(a.o_acc), obytes),
                        std::make_pair(static_cast<const void*>(a.lse_acc), lbytes),
                        std::make_pair(static_cast<const void*>(a.out), a.out ? outbytes : 0)})
    if (w.second && (overlap(w.first, w.second, a.q, qbytes) ||
                     overlap(w.first, w.second, a.k_rot, kbytes) ||
                     overlap(w.first, w.second, a.v, kbytes)))
      return RA_ERR_INVALID_ARG;
  if (overlap(a.o_acc, obytes, a.lse_acc, lbytes) ||
      (a.out && (overlap(a.out, outbytes, a.o_acc, obytes) ||
                 overlap(a.out, outbytes, a.lse_acc, lbytes))))
    return RA_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  // two slots per unit: two heads of a KV group (even G) or two consecutive query tiles of
  // one head (odd G)
  const int pair_q = G % 2;
  // each unit's rows lie in one segment: under the mask, q_split is a multiple of 128 rows
  // (256 with two query tiles per unit)
  if (two_seg && a.causal && a.q_split % (pair_q ? 256 : 128)) return RA_ERR_INVALID_ARG;
  const int n_qtiles = (Sq + 127) / 128;
  const int ppg = pair_q ? G : G / 2;
  const long long n_units =
      static_cast<long long>(pair_q ? (n_qtiles + 1) / 2 : n_qtiles) * B * Hkv * ppg;
  if (n_units > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return RA_ERR_UNSUPPORTED;

  DeviceState* ds = nullptr;
  ra_status rs = device_state(&ds);
  if (rs != RA_OK) return rs;
  // the (cos, sin) table of the query rows' positions (the keys arrive rotated): the cached
  // table of absolute positions, else one built here with one row per query row
  const int n0 = two_seg ? a.q_split : Sq;
  const long long rows_needed =
      std::max<long long>(static_cast<long long>(a.q_pos0) + n0,
                          two_seg ? static_cast<long long>(a.q_pos1) + (Sq - n0) : 0);
  const float2* tab_cached = nullptr;
  rs = cached_table(ds, a.rope_base, D, rows_needed, s, &tab_cached);
  if (rs != RA_OK) return rs;
  const size_t tab_bytes = tab_cached ? 256 : static_cast<size_t>(Sq) * (D / 2) * sizeof(float2);
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, tab_bytes, ds->pool, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync(workspace)");
  float2* tab = static_cast<float2*>(ws);
  if (!tab_cached) {
    ra::rope_table_kernel<<<grid_for(static_cast<long long>(n0) * (D / 2), 256, ds->num_sms),
                            256, 0, s>>>(tab, a.q_pos0, n0, D, a.rope_base);
    if (two_seg)
      ra::rope_table_kernel<<<grid_for(static_cast<long long>(Sq - n0) * (D / 2), 256,
                                       ds->num_sms), 256, 0, s>>>(
          tab + static_cast<size_t>(n0) * (D / 2), a.q_pos1, Sq - n0, D, a.rope_base);
  }
  CUtensorMap tq, tk, tv;
  rs = make_map(&tq, a.q, D, Sq, bhq, 128, q_rows);
  if (rs == RA_OK) rs = make_map(&tk, a.k_rot, D, Sk, bhk, 128, kv_rows);
  if (rs == RA_OK) rs = make_map(&tv, a.v, D, Sk, bhk, 128, kv_rows);
  if (rs == RA_OK) {
    ra::FwdParams p;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.tab = tab_cached ? tab_cached : tab;
    p.status = ds->status;
    p.wait_limit = g_wait_limit.load();
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.Sk = Sk;
    p.G = G;
    p.n_slots = 2;
    p.pair_q = pair_q;
    p.ppg = ppg;
    p.n_qtiles = n_qtiles;
    p.n_units = static_cast<int>(n_units);
    p.causal = a.causal ? 1 : 0;
    p.off = a.q_pos0 - a.k_pos0;  // query row i at q_pos0 + i, key j at k_pos0 + j
    p.off2 = two_seg ? a.q_pos1 - n0 - a.k_pos0 : p.off;  // row i >= n0 at q_pos1 + (i - n0)
    p.window = 0;
    // query row i sits at q_pos0 + i, or at q_pos1 + (i - n0) in the second segment
    p.q_tab_off = tab_cached ? a.q_pos0 : 0;
    p.q_split = n0;
    p.q_tab_off2 = tab_cached ? a.q_pos1 - n0 : 0;
    p.scale_log2 = kLog2e / std::sqrt(static_cast<float>(D));
    p.rope_base = a.rope_base;
    p.o_acc = a.o_acc;
    p.lse_acc = a.lse_acc;
    p.accumulate = (a.accumulate & RA_PARTIAL_ACCUMULATE) ? 1 : 0;
    p.dep_late = (a.accumulate & RA_PARTIAL_CHAINED) ? 1 : 0;
    p.acc_rows = acc_rows;
    rs = launch_attn(p, tq, tk, tv, tq, D, ds->num_sms, s);  // partial mode: no output map
  }
  cudaError_t ef = cudaFreeAsync(ws, s);
  if (rs == RA_OK && ef != cudaSuccess) rs = cuda_fail(ef, "cudaFreeAsync(workspace)");
  return rs;
}

// ------------------------------------------------------------------ decode
struct DecodeArgs {
  const void* q = nullptr;
  void* out = nullptr;
  const void* k_cache = nullptr;  // contiguous [B, Hkv, S_cache, D] or pool [nb, Hkv, page, D]
  const void* v_cache = nullptr;
  int B = 0, Hq = 0, Hkv = 0, D = 0;
  float rope_base = 0.f;
  int pos = 0;                    // every sequence's position when pos_arr is null
  const int* pos_arr = nullptr;   // device [B]
  int max_pos = 0;
  int window = 0;
  int n_splits = 0;
  int S_cache = 0;
  int page = 0;                   // > 0: paged pool
  const int* block_table = nullptr;
  int max_blocks = 0, num_blocks = 0;
  const void* k_new = nullptr;    // append (both or neither)
  const void* v_new = nullptr;
  bool noalloc = false;
  const char* who = "";
};

ra_status scratch_too_small(const char* who, size_t need) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                "%s: %zu bytes of partials exceed the %zu-byte scratch", who, need,
                kDecodeScratchBytes);
  return RA_ERR_UNSUPPORTED;
}

ra_status decode_impl(const DecodeArgs& a, cudaStream_t s) {
  const int B = a.B, Hq = a.Hq, Hkv = a.Hkv, D = a.D;
  if (!a.q || !a.k_cache || !a.v_cache || !a.out) return RA_ERR_INVALID_ARG;
  if (!aligned16(a.q) || !aligned16(a.k_cache) || !aligned16(a.v_cache) || !aligned16(a.out))
    return RA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || a.n_splits < 0 || a.window < 0 || a.max_pos < 0)
    return RA_ERR_INVALID_ARG;
  if (!a.pos_arr && a.pos < 0) return RA_ERR_INVALID_ARG;
  if (Hq % Hkv) return RA_ERR_INVALID_ARG;
  if (!(a.rope_base > 0.f) || !std::isfinite(a.rope_base)) return RA_ERR_INVALID_ARG;
  if ((a.k_new == nullptr) != (a.v_new == nullptr)) return RA_ERR_INVALID_ARG;
  if (a.k_new && (!aligned16(a.k_new) || !aligned16(a.v_new))) return RA_ERR_INVALID_ARG;
  const bool paged = a.page > 0;
  long long cap = 0;
  size_t cbytes = 0;
  if (paged) {
    if (64 % a.page || a.page < 8 || a.max_blocks < 1 || a.num_blocks < 1)
      return RA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(a.block_table) & 3u) return RA_ERR_INVALID_ARG;
    cap = static_cast<long long>(a.max_blocks) * a.page;
    cbytes = static_cast<size_t>(a.num_blocks) * Hkv * a.page * D * 2;
  } else {
    if (a.S_cache < 1) return RA_ERR_INVALID_ARG;
    cap = a.S_cache;
    cbytes = static_cast<size_t>(B) * Hkv * a.S_cache * D * 2;
  }
  if (cap > 0x7fffffffLL) return RA_ERR_INVALID_ARG;
  // per-sequence positions (and every paged or appending step) must lie inside the cache
  if ((a.pos_arr || paged || a.k_new) && a.max_pos >= cap) return RA_ERR_INVALID_ARG;
  if (a.max_pos > 0x7ffffffe) return RA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  const size_t qbytes = static_cast<size_t>(B) * Hq * D * 2;
  const size_t nbytes = static_cast<size_t>(B) * Hkv * D * 2;
  if (overlap(a.out, qbytes, a.q, qbytes) || overlap(a.out, qbytes, a.k_cache, cbytes) ||
      overlap(a.out, qbytes, a.v_cache, cbytes))
    return RA_ERR_INVALID_ARG;
  if (a.k_new) {
    for (const void* c : {a.k_cache, a.v_cache})
      if (overlap(c, cbytes, a.q, qbytes) || overlap(c, cbytes, a.k_new, nbytes) ||
          overlap(c, cbytes, a.v_new, nbytes))
        return RA_ERR_INVALID_ARG;
    if (overlap(a.k_cache, cbytes, a.v_cache, cbytes) || overlap(a.out, qbytes, a.k_new, nbytes) ||
        overlap(a.out, qbytes, a.v_new, nbytes))
      return RA_ERR_INVALID_ARG;
  }
  const int G = Hq / Hkv;
  const int hblocks = (G + 7) / 8;
  if (static_cast<long long>(B) * Hkv * hblocks > 65535) return RA_ERR_UNSUPPORTED;
  if (paged && static_cast<long long>(a.num_blocks) * Hkv > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;

  // rows a sequence attends at most (R) and the 64-aligned span the splits must cover
  const int L_max = static_cast<int>(std::min<long long>(cap, static_cast<long long>(a.max_pos) + 1));
  const int R = a.window > 0 ? std::min(a.window, L_max) : L_max;
  const int span = a.window > 0 ? R + 63 : L_max;
  auto cut = [&](int splits, int* chunk) {
    *chunk = ((span + splits - 1) / splits + 63) / 64 * 64;
    return (span + *chunk - 1) / *chunk;
  };
  int chunk = 0;
  if (a.noalloc && a.n_splits > 0) {
    // an explicit split count (as clamped by the rows) must fit the scratch; checked first
    const int req = cut(decode_splits(B, Hkv, G, span, 1, a.n_splits, paged), &chunk);
    if (decode_partials_bytes(B, Hq, D, req) > kDecodeScratchBytes)
      return scratch_too_small(a.who, decode_partials_bytes(B, Hq, D, req));
  }

  DeviceState* ds = nullptr;
  ra_status rs = device_state(&ds);
  if (rs != RA_OK) return rs;
  int splits = cut(decode_splits(B, Hkv, G, span, ds->num_sms, a.n_splits, paged), &chunk);
  void* scratch = nullptr;
  if (a.noalloc) {
    rs = decode_scratch(&scratch);
    if (rs != RA_OK) return rs;
    // automatic choice: the largest count up to the usual one whose partials fit
    while (splits > 1 && decode_partials_bytes(B, Hq, D, splits) > kDecodeScratchBytes)
      splits = cut(splits - 1, &chunk);
    if (decode_partials_bytes(B, Hq, D, splits) > kDecodeScratchBytes)
      return scratch_too_small(a.who, decode_partials_bytes(B, Hq, D, splits));
  }
  const size_t po_bytes =
      (static_cast<size_t>(B) * Hq * splits * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  const size_t pml_bytes = static_cast<size_t>(B) * Hq * splits * sizeof(float2);

  CUtensorMap tk, tv;
  if (paged) {
    const long long rows = static_cast<long long>(a.num_blocks) * Hkv;
    rs = make_map_dec(&tk, a.k_cache, D, a.page, rows, a.page);
    if (rs == RA_OK) rs = make_map_dec(&tv, a.v_cache, D, a.page, rows, a.page);
  } else {
    const long long bkv = static_cast<long long>(B) * Hkv;
    rs = make_map(&tk, a.k_cache, D, a.S_cache, bkv, 64);
    if (rs == RA_OK) rs = make_map(&tv, a.v_cache, D, a.S_cache, bkv, 64);
  }
  if (rs != RA_OK) return rs;

  void* ws = scratch;
  if (!a.noalloc) {
    cudaError_t e = cudaMallocFromPoolAsync(&ws, po_bytes + pml_bytes, ds->pool, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync(decode partials)");
  }
  ra::DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.part_o = static_cast<float*>(ws);
  p.part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + po_bytes);
  p.status = ds->status;
  p.wait_limit = g_wait_limit.load();
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = G;
  p.cap = static_cast<int>(cap);
  p.pos = a.pos;
  p.pos_arr = a.pos_arr;
  p.max_pos = a.max_pos;
  p.window = a.window;
  p.n_splits = splits;
  p.chunk = chunk;
  p.hblocks = hblocks;
  p.scale_log2 = kLog2e / std::sqrt(static_cast<float>(D));
  p.rope_base = a.rope_base;
  p.page = paged ? a.page : 0;
  p.block_table = a.block_table;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.num_blocks;
  p.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(a.v_new);
  p.k_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(a.k_cache));
  p.v_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(a.v_cache));
  p.S_cache = a.S_cache;
  const dim3 grid(static_cast<unsigned>(splits), static_cast<unsigned>(B * Hkv * hblocks));
  const int pi = prof_start(1, s);
  if (D == 64 && paged)
    ra::decode_split_kernel<64, true><<<grid, 160, ra::DecCfg<64>::SMEM, s>>>(tk, tv, p);
  else if (D == 64)
    ra::decode_split_kernel<64, false><<<grid, 160, ra::DecCfg<64>::SMEM, s>>>(tk, tv, p);
  else if (paged)
    ra::decode_split_kernel<128, true><<<grid, 160, ra::DecCfg<128>::SMEM, s>>>(tk, tv, p);
  else
    ra::decode_split_kernel<128, false><<<grid, 160, ra::DecCfg<128>::SMEM, s>>>(tk, tv, p);
  prof_stop(1, pi, s);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    // the combine may launch while the split kernel's last wave runs (it waits on the
    // device for the split grid to complete before reading the partials)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(B * Hq));
    cfg.blockDim = dim3(static_cast<unsigned>(D));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, ra::decode_combine_kernel, static_cast<const float*>(p.part_o),
                           static_cast<const float2*>(p.part_ml),
                           static_cast<__nv_bfloat16*>(a.out), splits, D);
  }
  if (e != cudaSuccess) rs = cuda_fail(e, "decode launch");
  if (!a.noalloc) {
    cudaError_t ef = cudaFreeAsync(ws, s);
    if (rs == RA_OK && ef != cudaSuccess) rs = cuda_fail(ef, "cudaFreeAsync(decode partials)");
  }
  return rs;
}

}  // namespace

extern "C" {

int rope_attn_version(void) { return 100; }

ra_status rope_attn_profile_enable(int enable) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof_on = enable != 0;
  g_prof_paused = false;
  g_prof[0].used = g_prof[1].used = 0;
  if (!g_prof_on) return RA_OK;
  // create the event pairs of the first kProfReserve launches of each kind now, on the
  // current device, so that profiled calls only record events
  constexpr size_t kProfReserve = 1024;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  for (ProfKind& pk : g_prof) {
    if (pk.device != dev) {
      for (auto& ev : pk.ev) { cudaEventDestroy(ev.first); cudaEventDestroy(ev.second); }
      pk.ev.clear();
      pk.device = dev;
    }
    while (pk.ev.size() < kProfReserve) {
      cudaEvent_t a, b;
      if ((e = cudaEventCreate(&a)) != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
      if ((e = cudaEventCreate(&b)) != cudaSuccess) {
        cudaEventDestroy(a);
        return cuda_fail(e, "cudaEventCreate");
      }
      pk.ev.emplace_back(a, b);
    }
  }
  return RA_OK;
}

ra_status rope_attn_profile_pause(int pause) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on) return RA_ERR_INVALID_ARG;
  g_prof_paused = pause != 0;
  return RA_OK;
}

ra_status rope_attn_profile_read(int which, double* total_ms, int* launches) {
  if ((which != 0 && which != 1) || !total_ms || !launches) return RA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  ProfKind& pk = g_prof[which];
  double sum = 0.0;
  for (size_t i = 0; i < pk.used; ++i) {
    cudaError_t e = cudaEventSynchronize(pk.ev[i].second);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pk.ev[i].first, pk.ev[i].second);
    if (e != cudaSuccess) return cuda_fail(e, "profile events");
    sum += ms;
  }
  *total_ms = sum;
  *launches = static_cast<int>(pk.used);
  pk.used = 0;
  return RA_OK;
}

long long rope_attn_set_wait_limit(long long limit) {
  if (limit < 0) return g_wait_limit.load();
  return g_wait_limit.exchange(limit);
}

const char* rope_attn_last_cuda_error(void) { return g_last_cuda_error; }

const char* rope_attn_status_string(int status) {
  switch (status) {
    case RA_OK: return "ok";
    case RA_ERR_INVALID_ARG: return "invalid argument";
    case RA_ERR_UNSUPPORTED: return "unsupported";
    case RA_ERR_CUDA: return g_last_cuda_error[0] ? g_last_cuda_error : "CUDA error";
    case RA_ERR_DEVICE_TIMEOUT: return "a kernel wait ran out (device timeout)";
    default: return "unknown status";
  }
}

ra_status rope_attn_get_device_status(ra_stream_t stream) {
  DeviceState* ds = nullptr;
  ra_status rs = device_state(&ds);
  if (rs != RA_OK) return rs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if ((e = cudaMemcpy(&v, ds->status, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "read status");
  const unsigned int zero = 0;
  if ((e = cudaMemcpy(ds->status, &zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e, "clear status");
  if (v & ra::kStatusArg) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "a per-sequence position or block-table entry was out of range; those "
                  "sequences were not computed");
    return RA_ERR_INVALID_ARG;
  }
  if (v & ra::kStatusLayout) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "kernel shared-memory base was not 1024-byte aligned; no work was done");
    return RA_ERR_CUDA;
  }
  return (v & ra::kStatusTimeout) ? RA_ERR_DEVICE_TIMEOUT : RA_OK;
}

ra_status rope_attn_rotate_rows(const void* x, void* x_rot, int B, int H, int S, int D,
                                float rope_base, int pos_offset, int x_rows, int out_rows,
                                ra_stream_t stream) {
  if (!x || !x_rot || !aligned16(x) || !aligned16(x_rot)) return RA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || S < 1 || D < 8 || D > 256 || D % 8) return RA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base) || pos_offset < 0) return RA_ERR_INVALID_ARG;
  if (static_cast<long long>(pos_offset) + S > 0x7fffffffLL) return RA_ERR_INVALID_ARG;
  if (x_rows < 0 || out_rows < 0) return RA_ERR_INVALID_ARG;
  if (x_rows == 0) x_rows = S;
  if (out_rows == 0) out_rows = S;
  if (x_rows < S || out_rows < S) return RA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * S;
  const long long heads = static_cast<long long>(B) * H;
  if (heads > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;  // the kernel counts heads in 32 bits
  const size_t xbytes = static_cast<size_t>((heads - 1) * x_rows + S) * D * 2;
  const size_t ybytes = static_cast<size_t>((heads - 1) * out_rows + S) * D * 2;
  // in place only with the same layout; otherwise the two must not share memory
  if (x == x_rot ? x_rows != out_rows : overlap(x, xbytes, x_rot, ybytes)) return RA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  ra_status rs = device_state(&ds);
  if (rs != RA_OK) return rs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ra::rope_rotate_kernel<false><<<rot_grid(ra::rope_tiles(heads, S, D), ds->num_sms),
                                  ra::kRotThreads, 0, s>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(x_rot), nullptr, rows, S, D, pos_offset,
      0, rope_base, x_rows, out_rows);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "rope_rotate launch");
}

ra_status rope_attn_rotate(const void* x, void* x_rot, int B, int H, int S, int D,
                           float rope_base, int pos_offset, ra_stream_t stream) {
  return rope_attn_rotate_rows(x, x_rot, B, H, S, D, rope_base, pos_offset, S, S, stream);
}


ra_status rope_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                        int Hkv, int Sq, int Sk, int D, float rope_base, int pos_offset,
                        int causal, ra_stream_t stream) {
  PrefillArgs a{q, k, v, out, nullptr, nullptr, 0, B, Hq, Hkv, Sq, Sk, D, rope_base,
                pos_offset, causal, 0};
  return prefill_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

ra_status rope_attn_fwd_partial(const void* q, const void* k_rot, const void* v, float* o_acc,
                                float* lse_acc, void* out, int B, int Hq, int Hkv, int Sq, int Sk,
                                int D, float rope_base, int q_pos0, int k_pos0, int causal,
                                int accumulate, int q_rows, int kv_rows, int acc_rows,
                                int q_split, int q_pos1, ra_stream_t stream) {
  PartialArgs a{q, k_rot, v, o_acc, lse_acc, out, B, Hq, Hkv, Sq, Sk, D, rope_base,
                q_pos0, k_pos0, causal, accumulate, q_rows, kv_rows, acc_rows, q_split, q_pos1};
  return partial_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

ra_status rope_attn_prefill(const void* q, const void* k, const void* v, void* out,
                            void* k_cache_rot, void* v_cache, int S_cache, int B, int Hq, int Hkv,
                            int Sq, int Sk, int D, float rope_base, int pos_offset, int causal,
                            int window, ra_stream_t stream) {
  PrefillArgs a{q, k, v, out, k_cache_rot, v_cache, S_cache, B, Hq, Hkv, Sq, Sk, D, rope_base,
                pos_offset, causal, window};
  return prefill_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

int rope_attn_decode_auto_splits(int B, int Hq, int Hkv, int Sk, int D, int pos) {
  (void)D;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sk < 1 || pos < 0 || Hq % Hkv) return 0;
  DeviceState* ds = nullptr;
  const int sms = (device_state(&ds) == RA_OK) ? ds->num_sms : 148;
  const int L = std::min(Sk, pos + 1);
  return decode_splits(B, Hkv, Hq / Hkv, L, sms, 0, false);
}

ra_status rope_attn_decode(const void* q, const void* k_cache_rot, const void* v_cache,
                           void* out, int B, int Hq, int Hkv, int Sk, int D, float rope_base,
                           int pos, int n_splits, ra_stream_t stream) {
  DecodeArgs a;
  a.q = q; a.out = out; a.k_cache = k_cache_rot; a.v_cache = v_cache;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.rope_base = rope_base;
  a.pos = pos; a.max_pos = pos; a.n_splits = n_splits; a.S_cache = Sk;
  a.who = "rope_attn_decode";
  return decode_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

ra_status rope_attn_decode_noalloc(const void* q, const void* k_cache_rot, const void* v_cache,
                                   void* out, int B, int Hq, int Hkv, int Sk, int D,
                                   float rope_base, int pos, int n_splits, ra_stream_t stream) {
  DecodeArgs a;
  a.q = q; a.out = out; a.k_cache = k_cache_rot; a.v_cache = v_cache;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.rope_base = rope_base;
  a.pos = pos; a.max_pos = pos; a.n_splits = n_splits; a.S_cache = Sk;
  a.noalloc = true;
  a.who = "rope_attn_decode_noalloc";
  return decode_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

ra_status rope_attn_decode_step(const void* q, const void* k_new, const void* v_new,
                                void* k_cache_rot, void* v_cache, void* out, const int* pos,
                                int B, int Hq, int Hkv, int S_cache, int D, float rope_base,
                                int max_pos, int window, int n_splits, ra_stream_t stream) {
  if (!pos) return RA_ERR_INVALID_ARG;
  DecodeArgs a;
  a.q = q; a.out = out; a.k_cache = k_cache_rot; a.v_cache = v_cache;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.rope_base = rope_base;
  a.pos_arr = pos; a.max_pos = max_pos; a.window = window; a.n_splits = n_splits;
  a.S_cache = S_cache;
  a.k_new = k_new; a.v_new = v_new;
  a.who = "rope_attn_decode_step";
  return decode_impl(a, reinterpret_cast<cudaStream_t>(stream));
}

ra_status rope_attn_decode_paged(const void* q, const void* k_new, const void* v_new,
                                 void* k_pool_rot, void* v_pool, const int* block_table,
                                 void* out, const int* pos, int B, int Hq, int Hkv, int D,
                                 int page_size, int max_blocks_per_seq, int num_blocks,
                                 float rope_base, int max_pos, int window, int n_splits,
                                 ra_stream_t stream) {
  if (!pos || !block_table || page_size < 1) return RA_ERR_INVALID_ARG;
  DecodeArgs a;
  a.q = q; a.out = out; a.k_cache = k_pool_rot; a.v_cache = v_pool;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.rope_base = rope_base;
  a.pos_arr = pos; a.max_pos = max_pos; a.window = window; a.n_splits = n_splits;
  a.page = page_size; a.block_table = block_table; a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_new = k_new; a.v_new = v_new;
  a.who = "rope_attn_decode_paged";
  return decode_impl(a, reinterpret_cast<cudaStream_t>(stream));
}


}  // extern "C"
