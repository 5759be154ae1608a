// pa_api.cu - the C ABI of the paged-attention library (declared in include/pa.h): argument
// validation, kernel selection, workspaces and the per-device error word.
//
// No call reads device data on the host or synchronises (pa_get_device_error and
// pa_release_workspaces excepted, as documented); launch sizes come from shapes only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "pa.h"
#include "pa_internal.h"
#include "pa_prefill_internal.h"

namespace {

// The error word of the device that loaded this module (one instance per device).
__device__ unsigned int g_pa_error_word;

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

typedef CUresult (*MemGetAddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
typedef CUresult (*PointerGetAttributesFn)(unsigned int, CUpointer_attribute *, void **, CUdeviceptr);
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Test hooks, read once per process: PA_TEST_WAIT_LIMIT_CYCLES shortens every wait on a copy;
// PA_TEST_STALL_COPIES makes a decode warp's first stage wait for 16 bytes that no copy
// delivers, so that the wait runs out, the kernel records PA_DEVERR_TIMEOUT and returns
// (1: every worker warp; 2: the odd-numbered worker warps only, so that the others finish their
// pieces and leave merge counters partly counted).  PA_TEST_STALL_CALLS limits the stall to the
// first n decode launches of the process (default: all of them).
struct TestHooks {
  long long wait_cycles = 2000000000ll;  // about one second at the 1965 MHz maximum SM clock
  int stall = 0;
  bool limited = false;                           // PA_TEST_STALL_CALLS given
  mutable std::atomic<long long> stall_calls{0};  // stalled launches left when limited
  TestHooks() {
    if (const char *v = std::getenv("PA_TEST_WAIT_LIMIT_CYCLES")) {
      const long long x = std::atoll(v);
      if (x > 0) wait_cycles = x;
    }
    if (const char *v = std::getenv("PA_TEST_STALL_COPIES")) {
      const int x = std::atoi(v);
      stall = (x == 1 || x == 2) ? x : 0;
    }
    if (const char *v = std::getenv("PA_TEST_STALL_CALLS")) {
      limited = true;
      stall_calls = std::atoll(v);
    }
  }
  // The stall mode of the next decode launch (0 once the limited number of launches is spent).
  int next_stall() const {
    if (!stall) return 0;
    if (!limited) return stall;
    return stall_calls.fetch_sub(1) > 0 ? stall : 0;
  }
};

const TestHooks &test_hooks() {
  static TestHooks h;
  return h;
}

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  unsigned int *err = nullptr;
  void *ws = nullptr;  // library-owned decode workspace
  size_t ws_bytes = 0;
};

std::mutex g_mu;
std::vector<DeviceState> g_devices;

// Merge counters sit at the start of a decode workspace, one per (sequence, kv head), and every
// completed call leaves them zero.  The regions after them move with the number of sequences,
// so a call with fewer sequences may write partial results where a later, larger call keeps
// counters.  For each workspace the library remembers how many leading bytes are known to hold
// zero counters and zeroes the rest (on the call's stream) before a call that needs more.
// How far a call goes: host-side argument checks only, every check (device memory, workspace
// size) without launching, the whole call, or the launch of a call whose every check has just
// passed with the same arguments (its device-memory queries are not repeated).
enum class CallMode { kHostChecks, kAllChecks, kLaunch, kLaunchChecked };

// Measurement aid (pa_set_decode_timeline): where decode launches record per-warp timestamps.
unsigned long long *g_timeline = nullptr;  // guarded by g_mu
long long g_timeline_warps = 0;

struct CleanRecord {
  const void *ws;
  size_t clean;
};
std::vector<CleanRecord> g_clean;  // guarded by g_mu

CleanRecord &clean_record(const void *ws) {
  for (auto &r : g_clean)
    if (r.ws == ws) return r;
  if (g_clean.size() >= 64) g_clean.erase(g_clean.begin());
  g_clean.push_back(CleanRecord{ws, 0});
  return g_clean.back();
}
MemGetAddressRangeFn g_mem_range = nullptr;
PointerGetAttributesFn g_ptr_attrs = nullptr;
EncodeTiledFn g_encode_tiled = nullptr;
bool g_mem_range_tried = false;

// Per-device set-up on first use: SM count and the address of the error word.
int device_state(DeviceState **out, int *dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  if ((int)g_devices.size() <= dev) g_devices.resize(dev + 1);
  DeviceState &st = g_devices[dev];
  if (!st.ready) {
    e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaGetSymbolAddress(reinterpret_cast<void **>(&st.err), g_pa_error_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    st.ready = true;
  }
  if (!g_mem_range_tried) {
    g_mem_range_tried = true;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_mem_range = reinterpret_cast<MemGetAddressRangeFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuPointerGetAttributes", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ptr_attrs = reinterpret_cast<PointerGetAttributesFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *out = &st;
  if (dev_out) *dev_out = dev;
  return PA_OK;
}

size_t elt_size(int dtype) {
  switch (dtype) {
    case PA_F32:
    case PA_I32:
      return 4;
    case PA_BF16:
    case PA_F16:
      return 2;
    case PA_I64:
      return 8;
    case PA_FP8_E4M3:
      return 1;
    default:
      return 0;
  }
}

const char *dtype_name(int d) {
  switch (d) {
    case PA_F32: return "fp32";
    case PA_BF16: return "bf16";
    case PA_F16: return "fp16";
    case PA_I32: return "int32";
    case PA_I64: return "int64";
    case PA_FP8_E4M3: return "fp8_e4m3";
    default: return "unknown";
  }
}

int check_tensor(const pa_tensor *t, const char *name, int ndim) {
  if (!t) return fail(PA_ERR_INVALID_ARG, "%s: NULL descriptor", name);
  if (t->ndim != ndim) return fail(PA_ERR_SHAPE, "%s: expected %d dims, got %d", name, ndim, t->ndim);
  if (elt_size(t->dtype) == 0) return fail(PA_ERR_DTYPE, "%s: unknown element type %d", name, t->dtype);
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return fail(PA_ERR_SHAPE, "%s: negative size in dim %d", name, i);
    if (t->stride[i] < 0) return fail(PA_ERR_LAYOUT, "%s: negative stride in dim %d", name, i);
  }
  return PA_OK;
}

int64_t numel(const pa_tensor *t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
  return n;
}

// The bytes from data to one past the last element the tensor addresses.
uint64_t extent_bytes(const pa_tensor *t) {
  if (numel(t) == 0) return 0;
  uint64_t last = 0;
  for (int i = 0; i < t->ndim; ++i) last += (uint64_t)(t->shape[i] - 1) * (uint64_t)t->stride[i];
  return (last + 1) * elt_size(t->dtype);
}

// Every byte the tensor addresses lies in one allocation of the current device.
int check_device_memory(const pa_tensor *t, const char *name, int dev) {
  const uint64_t ext = extent_bytes(t);
  if (ext == 0) return PA_OK;
  if (!t->data) return fail(PA_ERR_INVALID_ARG, "%s: NULL data pointer", name);
  const uint64_t p = (uint64_t)(uintptr_t)t->data;
  if (g_ptr_attrs) {
    // One driver query for the memory type, the device, managed or not and the allocation's
    // range (a pointer the driver does not know comes back with type 0).
    CUmemorytype type = (CUmemorytype)0;
    int ordinal = -1;
    CUdeviceptr start = 0;
    size_t size = 0;
    unsigned int managed = 0;  // the driver writes a one-byte bool into the low byte
    CUpointer_attribute which[5] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                    CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, CU_POINTER_ATTRIBUTE_RANGE_SIZE,
                                    CU_POINTER_ATTRIBUTE_IS_MANAGED};
    void *data[5] = {&type, &ordinal, &start, &size, &managed};
    if (g_ptr_attrs(5, which, data, (CUdeviceptr)(uintptr_t)t->data) == CUDA_SUCCESS) {
      const bool is_managed = (managed & 0xffu) != 0;
      if (type != CU_MEMORYTYPE_DEVICE && type != CU_MEMORYTYPE_UNIFIED && !is_managed)
        return fail(PA_ERR_LAYOUT, "%s: not device memory", name);
      if (!is_managed && type == CU_MEMORYTYPE_DEVICE && ordinal != dev)
        return fail(PA_ERR_LAYOUT, "%s: lives on device %d, current device is %d", name, ordinal, dev);
      if (size > 0 && p + ext > (uint64_t)start + size)
        return fail(PA_ERR_LAYOUT, "%s: addresses %llu bytes but its allocation ends after %llu", name,
                    (unsigned long long)ext, (unsigned long long)((uint64_t)start + size - p));
      return PA_OK;
    }
  }
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, t->data);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_LAYOUT, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(PA_ERR_LAYOUT, "%s: not device memory", name);
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
    return fail(PA_ERR_LAYOUT, "%s: lives on device %d, current device is %d", name, attr.device, dev);
  if (g_mem_range) {
    CUdeviceptr base = 0;
    size_t size = 0;
    // When the driver cannot name the allocation the pointer check above stands alone.
    if (g_mem_range(&base, &size, (CUdeviceptr)(uintptr_t)t->data) == CUDA_SUCCESS &&
        p + ext > (uint64_t)base + size)
      return fail(PA_ERR_LAYOUT, "%s: addresses %llu bytes but its allocation ends after %llu", name,
                  (unsigned long long)ext, (unsigned long long)((uint64_t)base + size - p));
  }
  return PA_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Strides of the dims [0, upto) multiplied by the element size are multiples of 16 bytes.
bool strides16(const pa_tensor *t, int upto) {
  const size_t e = elt_size(t->dtype);
  for (int i = 0; i < upto; ++i)
    if (((size_t)t->stride[i] * e) % 16 != 0) return false;
  return true;
}

struct CacheShape {
  int64_t num_blocks;
  int num_kv_heads, block_size, head_dim, dtype;
};

int check_caches(const pa_tensor *kc, const pa_tensor *vc, CacheShape *cs, bool allow_fp8 = false) {
  int rc;
  if ((rc = check_tensor(kc, "key_cache", 4)) || (rc = check_tensor(vc, "value_cache", 4))) return rc;
  for (int i = 0; i < 4; ++i)
    if (kc->shape[i] != vc->shape[i] || kc->stride[i] != vc->stride[i])
      return fail(PA_ERR_SHAPE, "key_cache and value_cache differ in shape or strides (dim %d)", i);
  if (kc->dtype != vc->dtype) return fail(PA_ERR_DTYPE, "key_cache and value_cache element types differ");
  if (kc->dtype == PA_FP8_E4M3 && !allow_fp8)
    return fail(PA_ERR_DTYPE, "FP8 caches need their scales: use the _fp8 entry points");
  if (kc->dtype != PA_F32 && kc->dtype != PA_BF16 && kc->dtype != PA_F16 && kc->dtype != PA_FP8_E4M3)
    return fail(PA_ERR_DTYPE, "caches must be fp32, bf16, fp16 or fp8_e4m3 (got %s)", dtype_name(kc->dtype));
  if (kc->stride[3] != 1 || kc->stride[2] != kc->shape[3])
    return fail(PA_ERR_LAYOUT, "caches: each (block, kv head) tile [block_size, head_dim] must be contiguous");
  if (!aligned16(kc->data) || !aligned16(vc->data) || !strides16(kc, 2))
    return fail(PA_ERR_LAYOUT, "caches: data and block/head strides must be 16-byte aligned");
  if (kc->shape[1] <= 0 || kc->shape[2] <= 0 || kc->shape[3] <= 0)
    return fail(PA_ERR_SHAPE, "caches: num_kv_heads, block_size and head_dim must be positive");
  if (kc->shape[1] > 0x7fffffff || kc->shape[2] > 0x7fffffff || kc->shape[3] > 0x7fffffff)
    return fail(PA_ERR_SHAPE, "caches: dimension too large");
  cs->num_blocks = kc->shape[0];
  cs->num_kv_heads = (int)kc->shape[1];
  cs->block_size = (int)kc->shape[2];
  cs->head_dim = (int)kc->shape[3];
  cs->dtype = kc->dtype;
  return PA_OK;
}

bool get_kernel(int dtype, int head_dim, int block_size, int group, bool tensor_cores,
                pa::DecodeKernel *k) {
  switch (dtype) {
    case PA_F32: return pa::decode_kernel_f32(head_dim, block_size, group, false, k);
    case PA_BF16: return pa::decode_kernel_bf16(head_dim, block_size, group, tensor_cores, k);
    case PA_F16: return pa::decode_kernel_f16(head_dim, block_size, group, tensor_cores, k);
    default: return false;
  }
}

// TMA descriptors of a cache, cached by everything they encode (the pools of a process are few).
struct MapKey {
  const void *ptr;
  int dtype, rows;
  int64_t shape[4], stride[4];
  bool operator==(const MapKey &o) const {
    if (ptr != o.ptr || dtype != o.dtype || rows != o.rows) return false;
    for (int i = 0; i < 4; ++i)
      if (shape[i] != o.shape[i] || stride[i] != o.stride[i]) return false;
    return true;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  uint64_t used;
};
std::vector<MapEntry> g_maps;
uint64_t g_map_clock = 0;

// The cache as a 5-D tensor (64 elements, block_size rows, head_dim / 64 column halves, kv heads,
// blocks) read in 128-byte swizzled boxes of 64 x `rows` x head_dim/64: one box brings a whole
// (rows x head_dim) tile, laid out in shared memory as [half][row][128 bytes].
// rows == 0 asks for the grouped view instead (caches whose blocks are kv heads x rows x
// head_dim contiguous, see grouped_view_ok): 64 elements, 8 rows, head_dim / 64 halves,
// block_size / 8 row groups, blocks x kv heads; one box brings a whole (block, kv head) tile laid
// out as [group of 8 rows][half][row][128 bytes], the operand layout of the tensor-core MMAs.
bool grouped_view_ok(const pa_tensor *t) {
  // (block, kv head) pairs are one coordinate of the view, a 32-bit TMA coordinate
  return t->stride[3] == 1 && t->stride[2] == t->shape[3] && t->stride[0] == t->shape[1] * t->stride[1] &&
         t->shape[2] % 8 == 0 && t->shape[0] * t->shape[1] <= 0x7fffffff;
}

int cache_map(const pa_tensor *t, int rows, CUtensorMap *out) {
  MapKey key;
  key.ptr = t->data;
  key.dtype = t->dtype;
  key.rows = rows;
  for (int i = 0; i < 4; ++i) {
    key.shape[i] = t->shape[i];
    key.stride[i] = t->stride[i];
  }
  std::lock_guard<std::mutex> lock(g_mu);
  for (auto &e : g_maps)
    if (e.key == key) {
      e.used = ++g_map_clock;
      *out = e.map;
      return PA_OK;
    }
  if (!g_encode_tiled) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t e = (cuuint64_t)elt_size(t->dtype);
  const cuuint64_t per128 = 128 / e;  // elements in one 128-byte swizzle span
  const cuuint64_t spans = (cuuint64_t)t->shape[3] / per128;
  cuuint64_t dims[5] = {per128, (cuuint64_t)t->shape[2], spans, (cuuint64_t)t->shape[1],
                        (cuuint64_t)t->shape[0]};
  cuuint64_t strides[4] = {(cuuint64_t)t->stride[2] * e, 128, (cuuint64_t)t->stride[1] * e,
                           (cuuint64_t)t->stride[0] * e};
  cuuint32_t box[5] = {(cuuint32_t)per128, (cuuint32_t)rows, (cuuint32_t)spans, 1, 1};
  if (rows == 0) {
    const cuuint64_t row_bytes = (cuuint64_t)t->shape[3] * e;
    const cuuint64_t g[5] = {per128, 8, spans, (cuuint64_t)t->shape[2] / 8,
                             (cuuint64_t)(t->shape[0] * t->shape[1])};
    const cuuint64_t st[4] = {row_bytes, 128, 8 * row_bytes, (cuuint64_t)t->stride[1] * e};
    const cuuint32_t bx[5] = {(cuuint32_t)per128, 8, (cuuint32_t)spans, (cuuint32_t)(t->shape[2] / 8), 1};
    for (int i = 0; i < 5; ++i) {
      dims[i] = g[i];
      box[i] = bx[i];
    }
    for (int i = 0; i < 4; ++i) strides[i] = st[i];
  }
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap map;
  const CUtensorMapDataType type = t->dtype == PA_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : t->dtype == PA_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = g_encode_tiled(
      &map, type,
      5, t->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_LAYOUT, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  if (g_maps.size() >= 16) {
    size_t old = 0;
    for (size_t i = 1; i < g_maps.size(); ++i)
      if (g_maps[i].used < g_maps[old].used) old = i;
    g_maps.erase(g_maps.begin() + old);
  }
  g_maps.push_back(MapEntry{key, map, ++g_map_clock});
  *out = map;
  return PA_OK;
}

// The prefill's query rows [tokens, heads, head_dim] as a 4-D tensor (64 elements, heads,
// tokens, head_dim / 64 halves) read in 128-byte swizzled boxes of 64 x G heads x 128/G tokens x
// halves: one box brings a tile's 128 rows (token-major, head fastest) laid out span-major,
// [half][row][128 bytes].  Tokens past the tensor read as zeros.
int query_map(const pa_tensor *q, int G, CUtensorMap *out) {
  if (!g_encode_tiled) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t e = 2;
  const cuuint64_t spans = (cuuint64_t)q->shape[2] / 64;
  const cuuint64_t dims[4] = {64, (cuuint64_t)q->shape[1], (cuuint64_t)q->shape[0], spans};
  const cuuint64_t strides[3] = {(cuuint64_t)q->stride[1] * e, (cuuint64_t)q->stride[0] * e, 128};
  const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G), (cuuint32_t)spans};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType type = q->dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = g_encode_tiled(out, type, 4, q->data, dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_LAYOUT, "cuTensorMapEncodeTiled failed for the query (%d)", (int)r);
  return PA_OK;
}

// Warps of one full wave of the device for a kernel (CTAs per SM x SMs x warps per CTA).
// The occupancy query is asked once per kernel and device (it costs host time on every call).
int default_workers(const pa::DecodeKernel &k, int num_sms) {
  struct Occ {
    const void *kernel;
    int dev, per_sm;
  };
  static std::vector<Occ> known;  // guarded by g_mu
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (const Occ &o : known)
      if (o.kernel == k.kernel && o.dev == dev) return o.per_sm * num_sms * k.warps_per_cta;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.kernel, k.threads_per_cta,
                                                    k.smem_bytes) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  } else {
    std::lock_guard<std::mutex> lock(g_mu);
    known.push_back(Occ{k.kernel, dev, per_sm});
  }
  return per_sm * num_sms * k.warps_per_cta;
}

// Workspace layout: counters [S*Hkv] u32 | pair_meta [S*Hkv] int2 | part_ml [(S*Hkv+W)*G*2] f32
//                   | part_o [(S*Hkv+W)*G*D] f32, each region 256-byte aligned.
struct WsLayout {
  size_t counters, pair_meta, part_ml, part_o, total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(int64_t S, int Hq, int Hkv, int D, int W) {
  WsLayout L;
  const size_t pairs = (size_t)S * (size_t)Hkv;
  const size_t segs = pairs + (size_t)W;
  const size_t G = (size_t)(Hq / Hkv);
  L.counters = 0;
  L.pair_meta = align256(pairs * 4);
  L.part_ml = L.pair_meta + align256(pairs * 8);
  L.part_o = L.part_ml + align256(segs * G * 2 * 4);
  L.total = L.part_o + align256(segs * G * (size_t)D * 4);
  return L;
}

// Shared-prefix pass: items of kPrefixItemTokens positions; its partial results follow the
// decode workspace: pre_ml [S*Hq*splits*2] f32 | pre_o [S*Hq*splits*D] f32.
#ifndef PA_PIECE_COST_16
#define PA_PIECE_COST_16 2  // split cost of a (sequence, kv head) start, 16-bit caches (chunks)
#endif
#ifndef PA_PIECE_COST_FP8
#define PA_PIECE_COST_FP8 4  // the same, FP8 caches
#endif
#ifndef PA_PIECE_COST_SHARED
#define PA_PIECE_COST_SHARED 2  // the same, shared-prefix decode (each piece also merges the
                                // prefix pass's partial results)
#endif
constexpr int kMaxPieceCost = PA_PIECE_COST_16 > PA_PIECE_COST_FP8
                                  ? (PA_PIECE_COST_16 > PA_PIECE_COST_SHARED ? PA_PIECE_COST_16 : PA_PIECE_COST_SHARED)
                                  : (PA_PIECE_COST_FP8 > PA_PIECE_COST_SHARED ? PA_PIECE_COST_FP8 : PA_PIECE_COST_SHARED);

#ifndef PA_PREFIX_ITEM_TOKENS
#define PA_PREFIX_ITEM_TOKENS 512
#endif
// Positions of one prefix-pass item (a multiple of the prefill kernel's 128-position kv tile):
// each item leaves one partial result per (member, query head) for the decode to merge.  On the
// 128-sequence shared-prefix batch (1024-position prompt) the cascade took 64.1 us with items of
// 256 positions, 63.0 with 512 (half the CTAs, each over four kv tiles, leave SMs to the decode
// sooner, and each merge takes two prefix pieces instead of four), 67.7 with 1024.
constexpr int kPrefixItemTokens = PA_PREFIX_ITEM_TOKENS;

struct PrefixLayout {
  size_t pre_ml, pre_o, total;
  int splits;
};

PrefixLayout prefix_layout(size_t start, int64_t S, int Hq, int D, int64_t max_blocks,
                           int block_size) {
  PrefixLayout P;
  const int64_t max_len = max_blocks * block_size;
  P.splits = (int)((max_len + kPrefixItemTokens - 1) / kPrefixItemTokens);
  if (P.splits < 1) P.splits = 1;
  const size_t slots = (size_t)S * (size_t)Hq * (size_t)P.splits;
  P.pre_ml = align256(start);
  P.pre_o = P.pre_ml + align256(slots * 2 * 4);
  P.total = P.pre_o + align256(slots * (size_t)D * 4);
  return P;
}

#ifndef PA_PREFIX_SM_DIVISOR
#define PA_PREFIX_SM_DIVISOR 1
#endif
// The prefix pass runs on at most 1/PA_PREFIX_SM_DIVISOR of the SMs (its persistent CTAs take
// the items in rounds); the decode, launched to overlap it, streams the suffixes on whatever SMs
// are free and waits for the pass only to merge.  Each item is a chain of dependent hand-offs,
// so fewer CTAs lengthen the pass more than the decode gains: on the 128-sequence shared-prefix
// batch the cascade took 64.0 us with every SM, 69.1 / 75.5 / 94.2 us with a third, a quarter,
// a sixth (the decode then sized to the SMs left).
int prefix_pass_ctas(int64_t S, int64_t NG, int num_kv_heads, int splits, int tokens_per_tile,
                     int num_sms) {
  if (NG <= 0) return 0;
  const int64_t items = ((S + tokens_per_tile - 1) / tokens_per_tile + NG) * num_kv_heads * (int64_t)splits;
  int64_t cap = num_sms / PA_PREFIX_SM_DIVISOR;
  if (cap < 1) cap = 1;
  return (int)(items < cap ? items : cap);
}

bool prefix_pass_kernel(const CacheShape &cs, int D, int G, int block_size, pa::PrefillKernel *k) {
  return cs.dtype == PA_BF16 ? pa::prefill_kernel_bf16(D, block_size, G, k)
                             : pa::prefill_kernel_f16(D, block_size, G, k);
}

// The prefix pass of pa_decode_shared_prefix: the prefill kernel over every group's members
// (their decode queries as consecutive query rows) and its shared prefix, storing partial
// results for the decode to merge, on `ctas` persistent CTAs.
int launch_prefix_pass(const pa::DecodeArgs &d, const pa_tensor *query, const pa_tensor *key_cache,
                       const pa_tensor *value_cache, const pa_tensor *group_start,
                       const CacheShape &cs, int D, int G, int block_size, int ctas,
                       cudaStream_t st) {
  int rc;
  pa::PrefillKernel k;
  if (!prefix_pass_kernel(cs, D, G, block_size, &k))
    return fail(PA_ERR_CUDA, "could not prepare the prefix pass: %s", cudaGetErrorString(cudaGetLastError()));
  pa::PrefillMaps maps;
  const pa_tensor *kc = key_cache, *vc = value_cache;
  const bool grouped = grouped_view_ok(kc) && grouped_view_ok(vc);
  const int rows = grouped ? 0 : k.tma_rows;
  if ((rc = cache_map(kc, rows, &maps.k)) || (rc = cache_map(vc, rows, &maps.v)) ||
      (rc = query_map(query, G, &maps.q)))
    return rc;
  const int64_t S = d.num_seqs;
  const int64_t NG = group_start->shape[0] - 1;
  if (NG <= 0 || ctas <= 0) return PA_OK;
  pa::PrefillArgs a = {};
  a.out = nullptr;
  a.out_dtype = PA_F32;
  a.query = query->data;
  a.q_t = query->stride[0];
  a.q_h = query->stride[1];
  a.block_tables = d.block_tables;
  a.bt_s = d.bt_s;
  a.context_lens = d.context_lens;
  a.query_start = nullptr;
  a.num_seqs = d.num_seqs;
  a.num_kv_heads = d.num_kv_heads;
  a.max_blocks = d.max_blocks;
  a.num_blocks = d.num_blocks;
  a.num_tokens = S;
  a.scale_log2 = d.scale_log2;
  a.err = d.err;
  a.wait_cycles = d.wait_cycles;
  a.grouped_maps = grouped ? 1 : 0;
  a.group_start = static_cast<const int32_t *>(group_start->data);
  a.prefix_lens = d.prefix_lens;
  a.num_groups = (int)NG;
  a.pre_kv = kPrefixItemTokens / 128;
  a.pre_splits = d.pre_splits;
  a.pre_o = const_cast<float *>(d.pre_o);
  a.pre_ml = const_cast<float *>(d.pre_ml);
  cudaError_t e = k.launch(a, &maps, ctas, st);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "prefix pass launch");
}

int decode_impl(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                const pa_tensor *value_cache, const pa_tensor *block_tables,
                const pa_tensor *context_lens, float scale, int32_t block_size,
                int32_t num_kv_heads, int32_t num_workers, uint32_t flags, void *workspace,
                size_t workspace_bytes, bool library_workspace, void *stream,
                CallMode mode = CallMode::kLaunch, const pa_tensor *k_scale = nullptr,
                const pa_tensor *v_scale = nullptr, const pa_tensor *group_start = nullptr,
                const pa_tensor *prefix_lens = nullptr, const pa::CacheWriteArgs *step = nullptr) {
  int rc;
  CacheShape cs;
  const bool fp8 = k_scale != nullptr;
  const bool shared = group_start != nullptr;
  if ((rc = check_caches(key_cache, value_cache, &cs, fp8))) return rc;
  if (fp8 && cs.dtype != PA_FP8_E4M3) return fail(PA_ERR_DTYPE, "pa_decode_fp8 needs fp8_e4m3 caches");
  if ((rc = check_tensor(query, "query", 3)) || (rc = check_tensor(out, "out", 3)) ||
      (rc = check_tensor(block_tables, "block_tables", 2)) ||
      (rc = check_tensor(context_lens, "context_lens", 1)))
    return rc;
  if (flags & ~(PA_DECODE_SEPARATE_REDUCE | PA_DECODE_CUDA_CORES | PA_DECODE_OVERLAP_PREVIOUS))
    return fail(PA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (num_workers < 0) return fail(PA_ERR_INVALID_ARG, "num_workers must be >= 0");
  if (block_size != cs.block_size)
    return fail(PA_ERR_SHAPE, "block_size %d does not match the cache's %d", block_size, cs.block_size);
  if (num_kv_heads != cs.num_kv_heads)
    return fail(PA_ERR_SHAPE, "num_kv_heads %d does not match the cache's %d", num_kv_heads, cs.num_kv_heads);
  const int64_t S = query->shape[0];
  const int64_t Hq = query->shape[1];
  const int D = cs.head_dim;
  if (query->shape[2] != D) return fail(PA_ERR_SHAPE, "query head_dim %lld != cache head_dim %d", (long long)query->shape[2], D);
  if (out->shape[0] != S || out->shape[1] != Hq || out->shape[2] != D)
    return fail(PA_ERR_SHAPE, "out must be [num_seqs, num_heads, head_dim] like query");
  if (block_tables->shape[0] != S || context_lens->shape[0] != S)
    return fail(PA_ERR_SHAPE, "block_tables and context_lens need one row per sequence");
  if (fp8) {
    if (query->dtype != PA_BF16 && query->dtype != PA_F16)
      return fail(PA_ERR_DTYPE, "with FP8 caches the query must be bf16 or fp16");
    if (out->dtype != PA_F32 && out->dtype != query->dtype)
      return fail(PA_ERR_DTYPE, "out must be fp32 or the query's element type");
    if ((rc = check_tensor(k_scale, "k_scale", 1)) || (rc = check_tensor(v_scale, "v_scale", 1)))
      return rc;
    if (k_scale->dtype != PA_F32 || v_scale->dtype != PA_F32)
      return fail(PA_ERR_DTYPE, "k_scale and v_scale must be fp32");
    if (k_scale->shape[0] != num_kv_heads || v_scale->shape[0] != num_kv_heads)
      return fail(PA_ERR_SHAPE, "k_scale and v_scale need one value per kv head");
    if ((k_scale->stride[0] != 1 || v_scale->stride[0] != 1) && num_kv_heads > 1)
      return fail(PA_ERR_LAYOUT, "k_scale and v_scale must be contiguous");
    if (flags & PA_DECODE_CUDA_CORES)
      return fail(PA_ERR_UNSUPPORTED, "FP8 caches are read by the tensor-core kernel only");
    if (cs.head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "FP8 caches: head_dim %d (built: 128)", cs.head_dim);
  } else {
    if (query->dtype != cs.dtype) return fail(PA_ERR_DTYPE, "query must have the caches' element type");
    if (out->dtype != PA_F32 && out->dtype != cs.dtype)
      return fail(PA_ERR_DTYPE, "out must be fp32 or the caches' element type");
  }
  if (block_tables->dtype != PA_I32 || context_lens->dtype != PA_I32)
    return fail(PA_ERR_DTYPE, "block_tables and context_lens must be int32");
  if (Hq <= 0 && S > 0) return fail(PA_ERR_SHAPE, "num_heads must be positive");
  if (Hq % num_kv_heads != 0) return fail(PA_ERR_SHAPE, "num_heads %lld is not a multiple of num_kv_heads %d", (long long)Hq, num_kv_heads);
  const int G = (int)(Hq / num_kv_heads);
  if (D != 64 && D != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d (built: 64, 128)", D);
  if (block_size != 8 && block_size != 16 && block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (built: 8, 16, 32)", block_size);
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per kv head %d (built: 1, 2, 4, 8)", G);
  if (query->stride[2] != 1 || out->stride[2] != 1)
    return fail(PA_ERR_LAYOUT, "query and out need a contiguous head_dim");
  if (!aligned16(query->data) || !strides16(query, 2) || !aligned16(out->data) || !strides16(out, 2))
    return fail(PA_ERR_LAYOUT, "query/out: data and sequence/head strides must be 16-byte aligned");
  if (block_tables->stride[1] != 1 && block_tables->shape[1] > 1)
    return fail(PA_ERR_LAYOUT, "block_tables rows must be contiguous");
  if (context_lens->stride[0] != 1 && S > 1) return fail(PA_ERR_LAYOUT, "context_lens must be contiguous");
  if (S > 0x7fffffff || block_tables->shape[1] * block_size > 0x7fffffff)
    return fail(PA_ERR_SHAPE, "too many sequences or too long a block table");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  if (shared) {
    if (!prefix_lens) return fail(PA_ERR_INVALID_ARG, "prefix_lens is required");
    if ((rc = check_tensor(group_start, "group_start", 1)) || (rc = check_tensor(prefix_lens, "prefix_lens", 1)))
      return rc;
    if (group_start->dtype != PA_I32 || prefix_lens->dtype != PA_I32)
      return fail(PA_ERR_DTYPE, "group_start and prefix_lens must be int32");
    if (group_start->shape[0] < 1 || prefix_lens->shape[0] != S)
      return fail(PA_ERR_SHAPE, "group_start needs num_groups + 1 entries and prefix_lens one per sequence");
    if ((group_start->stride[0] != 1 && group_start->shape[0] > 1) || (prefix_lens->stride[0] != 1 && S > 1))
      return fail(PA_ERR_LAYOUT, "group_start and prefix_lens must be contiguous");
    if (cs.dtype != PA_BF16 && cs.dtype != PA_F16)
      return fail(PA_ERR_UNSUPPORTED, "shared prefixes are built for bf16 and fp16 caches");
    if (group_start->shape[0] - 1 > 0x7fffffff) return fail(PA_ERR_SHAPE, "too many groups");
  }
  // a worker counts its share's chunks in 32 bits: at most 2e9 chunks of 16 positions a step
  // (counting each (sequence, kv head) start at the largest piece cost)
  if ((double)S * num_kv_heads * ((double)block_tables->shape[1] * block_size / 16 + 1 + kMaxPieceCost) > 2.0e9)
    return fail(PA_ERR_SHAPE, "step too large for the work split");
  if (S == 0 || mode == CallMode::kHostChecks) return PA_OK;
  DeviceState *ds;
  int dev;
  if ((rc = device_state(&ds, &dev))) return rc;
  if (mode != CallMode::kLaunchChecked) {
  if (shared && ((rc = check_device_memory(group_start, "group_start", dev)) ||
                 (rc = check_device_memory(prefix_lens, "prefix_lens", dev))))
    return rc;
  if ((rc = check_device_memory(key_cache, "key_cache", dev)) ||
      (rc = check_device_memory(value_cache, "value_cache", dev)) ||
      (rc = check_device_memory(query, "query", dev)) || (rc = check_device_memory(out, "out", dev)) ||
      (rc = check_device_memory(block_tables, "block_tables", dev)) ||
      (rc = check_device_memory(context_lens, "context_lens", dev)))
    return rc;
  if (fp8 && ((rc = check_device_memory(k_scale, "k_scale", dev)) ||
              (rc = check_device_memory(v_scale, "v_scale", dev))))
    return rc;
  }

  pa::DecodeKernel k;
  const bool tensor_cores = cs.dtype != PA_F32 && !(flags & PA_DECODE_CUDA_CORES);
  const bool got = fp8 ? pa::decode_kernel_fp8(query->dtype, D, block_size, G, &k)
                       : get_kernel(cs.dtype, D, block_size, G, tensor_cores, &k);
  if (!got)
    return fail(PA_ERR_CUDA, "could not prepare the decode kernel: %s", cudaGetErrorString(cudaGetLastError()));
  pa::TmaMaps maps;
  if (k.tma_rows > 0) {
    if ((rc = cache_map(key_cache, k.tma_rows, &maps.k)) || (rc = cache_map(value_cache, k.tma_rows, &maps.v)))
      return rc;
  }
  // shared prefixes: the SMs the prefix pass leaves to the decode
  int prefix_ctas = 0;
  if (shared) {
    pa::PrefillKernel pk;
    if (!prefix_pass_kernel(cs, D, G, block_size, &pk))
      return fail(PA_ERR_CUDA, "could not prepare the prefix pass: %s", cudaGetErrorString(cudaGetLastError()));
    const int64_t max_len = block_tables->shape[1] * block_size;
    const int splits = (int)((max_len + kPrefixItemTokens - 1) / kPrefixItemTokens);
    prefix_ctas = prefix_pass_ctas(S, group_start->shape[0] - 1, num_kv_heads, splits < 1 ? 1 : splits,
                                   pk.tokens_per_tile, ds->num_sms);
  }
  // (the decode is sized to the SMs left when the pass takes at most half of them)
  const int decode_sms = k.tma_rows > 0 && 2 * prefix_ctas <= ds->num_sms ? ds->num_sms - prefix_ctas : ds->num_sms;
  const int W = num_workers > 0 ? num_workers : default_workers(k, decode_sms);
  // The split's cost of a (sequence, kv head) start, in chunks: what a warp spends once per
  // piece (query rows, partial result, ticket, merge).  Per-warp timings of the Llama-shaped
  // step put it near one chunk's time with 16-bit caches and two to three with FP8 (whose
  // chunks take less time); once the workers' per-chunk chain was cut, the fastest measured
  // became 2 for 16-bit caches (against 0, 1, 3) and 4 for FP8 (against 2, 3).
  const int piece_cost = k.tma_rows == 0 ? 0
                         : shared       ? PA_PIECE_COST_SHARED
                         : fp8          ? PA_PIECE_COST_FP8
                                        : PA_PIECE_COST_16;
  // worker_of() multiplies a position by W in 64 bits; a worker counts its share's chunks in 32
  const double chunks = (double)S * num_kv_heads *
                        ((double)block_tables->shape[1] * block_size / k.chunk_tokens + 1 + piece_cost);
  if (chunks * (double)W > 4.0e18 || chunks > 2.0e9)
    return fail(PA_ERR_SHAPE, "step too large for the work split");
  const WsLayout L = ws_layout(S, (int)Hq, num_kv_heads, D, W);
  const PrefixLayout PL = prefix_layout(L.total, S, (int)Hq, D, block_tables->shape[1], block_size);
  const size_t need = shared ? PL.total : L.total;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode == CallMode::kAllChecks) {  // everything a launch would check, nothing launched
    if (!library_workspace && (!workspace || workspace_bytes < need))
      return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!library_workspace && ((uintptr_t)workspace & 255u) != 0)
      return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    return PA_OK;
  }
  if (library_workspace) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (ds->ws_bytes < need) {
      cudaError_t e;
      if (ds->ws) {
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize (workspace growth)");
        cudaFree(ds->ws);
        clean_record(ds->ws).clean = 0;
        ds->ws = nullptr;
        ds->ws_bytes = 0;
      }
      const size_t want = need + need / 4;
      e = cudaMalloc(&ds->ws, want);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(decode workspace)");
      e = cudaMemsetAsync(ds->ws, 0, want, st);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(decode workspace)");
      ds->ws_bytes = want;
      clean_record(ds->ws).clean = want;
    }
    workspace = ds->ws;
    workspace_bytes = ds->ws_bytes;
  } else {
    if (!workspace || workspace_bytes < need)
      return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (((uintptr_t)workspace & 255u) != 0) return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  {
    const size_t counter_bytes = (size_t)S * (size_t)num_kv_heads * 4;
    std::lock_guard<std::mutex> lock(g_mu);
    CleanRecord &rec = clean_record(workspace);
    if (rec.clean < counter_bytes) {
      cudaError_t e = cudaMemsetAsync(static_cast<char *>(workspace) + rec.clean, 0,
                                      counter_bytes - rec.clean, st);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(merge counters)");
    }
    rec.clean = counter_bytes;
  }

  pa::DecodeArgs a = {};
  a.out = out->data;
  a.out_dtype = out->dtype;
  a.out_s = out->stride[0];
  a.out_h = out->stride[1];
  a.query = query->data;
  a.q_s = query->stride[0];
  a.q_h = query->stride[1];
  a.q_heads_contiguous = (query->stride[1] == D) ? 1 : 0;
  a.key_cache = key_cache->data;
  a.value_cache = value_cache->data;
  a.kv_blk = key_cache->stride[0];
  a.kv_head = key_cache->stride[1];
  a.block_tables = static_cast<const int32_t *>(block_tables->data);
  a.bt_s = block_tables->stride[0];
  a.context_lens = static_cast<const int32_t *>(context_lens->data);
  a.num_seqs = (int)S;
  a.num_kv_heads = num_kv_heads;
  a.max_blocks = (int)block_tables->shape[1];
  a.num_blocks = cs.num_blocks;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.num_workers = W;
  a.piece_cost = piece_cost;
  char *ws = static_cast<char *>(workspace);
  a.counters = reinterpret_cast<unsigned int *>(ws + L.counters);
  a.pair_meta = reinterpret_cast<int2 *>(ws + L.pair_meta);
  a.part_ml = reinterpret_cast<float *>(ws + L.part_ml);
  a.part_o = reinterpret_cast<float *>(ws + L.part_o);
  a.err = ds->err;
  a.k_scale = fp8 ? static_cast<const float *>(k_scale->data) : nullptr;
  a.v_scale = fp8 ? static_cast<const float *>(v_scale->data) : nullptr;
  a.separate_reduce = (flags & PA_DECODE_SEPARATE_REDUCE) ? 1 : 0;
  a.wait_cycles = test_hooks().wait_cycles;
  a.test_stall = test_hooks().next_stall();
  {
    std::lock_guard<std::mutex> lock(g_mu);
    a.timeline = g_timeline;
    a.timeline_warps = g_timeline_warps;
  }
  bool overlap = (flags & PA_DECODE_OVERLAP_PREVIOUS) != 0;
  if (step) {
    a.fused = 1;
    a.step = *step;
  }
  if (shared) {
    a.prefix_lens = static_cast<const int32_t *>(prefix_lens->data);
    a.pre_ml = reinterpret_cast<float *>(ws + PL.pre_ml);
    a.pre_o = reinterpret_cast<float *>(ws + PL.pre_o);
    a.pre_splits = PL.splits;
    a.pre_kv_tokens = kPrefixItemTokens;
    if ((rc = launch_prefix_pass(a, query, key_cache, value_cache, group_start, cs, D, G,
                                 block_size, prefix_ctas, st)))
      return rc;
    overlap = true;  // the decode runs while the prefix pass does
    // the tensor-core decode streams at once (the pass is stream-ordered after the caches'
    // writers) and waits for the pass only before merging its partial results
    a.prefix_overlap = k.tma_rows > 0 ? 1 : 0;
  }
  const int ctas = (W + k.warps_per_cta - 1) / k.warps_per_cta;  // warps_per_cta workers each
  cudaError_t e = k.launch(a, &maps, ctas, overlap, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if (a.separate_reduce) {
    e = k.launch_reduce(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return PA_OK;
}

}  // namespace

namespace pa {

// Helpers for the allocation-free entry point (pa_noalloc.cu).
void set_last_error(const char *msg) { g_last_error = msg; }

size_t decode_scratch_need(const pa_tensor *query, const pa_tensor *key_cache, int32_t block_size,
                           int32_t num_kv_heads) {
  if (!query || !key_cache || query->ndim != 3 || key_cache->ndim != 4 || num_kv_heads <= 0 ||
      query->shape[1] % num_kv_heads != 0)
    return 0;
  DeviceState *ds;
  if (device_state(&ds, nullptr) != PA_OK) return 0;
  DecodeKernel k;
  const int D = (int)key_cache->shape[3];
  const int G = (int)(query->shape[1] / num_kv_heads);
  if (!get_kernel(key_cache->dtype, D, block_size, G, key_cache->dtype != PA_F32, &k)) return 0;
  return ws_layout(query->shape[0], (int)query->shape[1], num_kv_heads, D,
                   default_workers(k, ds->num_sms)).total;
}

int decode_into(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                const pa_tensor *value_cache, const pa_tensor *block_tables,
                const pa_tensor *context_lens, float scale, int32_t block_size,
                int32_t num_kv_heads, void *workspace, size_t workspace_bytes, void *stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, 0, 0u, workspace, workspace_bytes, false, stream);
}

}  // namespace pa

namespace {

int write_impl(const pa_tensor *key, const pa_tensor *value, const pa_tensor *key_cache,
               const pa_tensor *value_cache, const pa_tensor *slot_mapping, void *stream,
               CallMode mode, pa::CacheWriteArgs *prepared = nullptr) {
  int rc;
  CacheShape cs;
  if ((rc = check_caches(key_cache, value_cache, &cs))) return rc;
  if ((rc = check_tensor(key, "key", 3)) || (rc = check_tensor(value, "value", 3)) ||
      (rc = check_tensor(slot_mapping, "slot_mapping", 1)))
    return rc;
  const int64_t T = key->shape[0];
  for (int i = 0; i < 3; ++i)
    if (value->shape[i] != key->shape[i]) return fail(PA_ERR_SHAPE, "key and value shapes differ");
  if (key->shape[1] != cs.num_kv_heads || key->shape[2] != cs.head_dim)
    return fail(PA_ERR_SHAPE, "key/value must be [num_tokens, num_kv_heads, head_dim] of the cache");
  if (slot_mapping->shape[0] != T) return fail(PA_ERR_SHAPE, "slot_mapping needs one slot per token");
  if (key->dtype != cs.dtype || value->dtype != cs.dtype)
    return fail(PA_ERR_DTYPE, "key/value must have the caches' element type");
  if (slot_mapping->dtype != PA_I64) return fail(PA_ERR_DTYPE, "slot_mapping must be int64");
  if (key->stride[2] != 1 || value->stride[2] != 1 || (slot_mapping->stride[0] != 1 && T > 1))
    return fail(PA_ERR_LAYOUT, "key/value need a contiguous head_dim and slot_mapping unit stride");
  if (!aligned16(key->data) || !aligned16(value->data) || !strides16(key, 2) || !strides16(value, 2))
    return fail(PA_ERR_LAYOUT, "key/value: data and token/head strides must be 16-byte aligned");
  if (T == 0 || mode == CallMode::kHostChecks) return PA_OK;
  DeviceState *ds;
  int dev;
  if ((rc = device_state(&ds, &dev))) return rc;
  if (mode != CallMode::kLaunchChecked &&
      ((rc = check_device_memory(key_cache, "key_cache", dev)) ||
       (rc = check_device_memory(value_cache, "value_cache", dev)) ||
       (rc = check_device_memory(key, "key", dev)) || (rc = check_device_memory(value, "value", dev)) ||
       (rc = check_device_memory(slot_mapping, "slot_mapping", dev))))
    return rc;
  const size_t e = elt_size(cs.dtype);
  pa::CacheWriteArgs a;
  a.key = static_cast<const char *>(key->data);
  a.value = static_cast<const char *>(value->data);
  a.k_tok = key->stride[0] * (int64_t)e;
  a.k_head = key->stride[1] * (int64_t)e;
  a.v_tok = value->stride[0] * (int64_t)e;
  a.v_head = value->stride[1] * (int64_t)e;
  a.key_cache = static_cast<char *>(key_cache->data);
  a.value_cache = static_cast<char *>(value_cache->data);
  a.c_blk = key_cache->stride[0] * (int64_t)e;
  a.c_head = key_cache->stride[1] * (int64_t)e;
  a.row_bytes = (int)(cs.head_dim * e);
  a.slots = static_cast<const int64_t *>(slot_mapping->data);
  a.num_tokens = T;
  a.num_kv_heads = cs.num_kv_heads;
  a.block_size = cs.block_size;
  a.num_slots = cs.num_blocks * cs.block_size;
  a.err = ds->err;
  if (a.row_bytes % 16 != 0) return fail(PA_ERR_UNSUPPORTED, "head_dim * element size must be a multiple of 16 bytes");
  if (prepared) *prepared = a;
  if (mode == CallMode::kAllChecks) return PA_OK;
  cudaError_t err = pa::launch_reshape_and_cache(a, ds->num_sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? PA_OK : cuda_fail(err, "reshape_and_cache launch");
}

// Device address through which a kernel on `dev` reaches t's data: device (or managed) memory
// of that device, or pinned host memory mapped into the device's address space.  Pageable
// host memory is refused.  The extent is checked for device allocations only.
int device_address(const pa_tensor *t, const char *name, int dev, void **addr) {
  *addr = t->data;
  if (extent_bytes(t) == 0) return PA_OK;
  if (!t->data) return fail(PA_ERR_INVALID_ARG, "%s: NULL data pointer", name);
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, t->data);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_LAYOUT, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (attr.type == cudaMemoryTypeHost) {
    if (!attr.devicePointer)
      return fail(PA_ERR_LAYOUT, "%s: pinned host memory not mapped into the device", name);
    *addr = attr.devicePointer;
    return PA_OK;
  }
  return check_device_memory(t, name, dev);
}

int copy_blocks_impl(const pa_tensor *src_k, const pa_tensor *src_v, const pa_tensor *dst_k,
                     const pa_tensor *dst_v, const pa_tensor *block_mapping, bool host_allowed,
                     void *stream) {
  int rc;
  CacheShape s, d;
  if ((rc = check_caches(src_k, src_v, &s, true))) return rc;
  if ((rc = check_caches(dst_k, dst_v, &d, true))) return rc;
  if (s.dtype != d.dtype || s.num_kv_heads != d.num_kv_heads || s.block_size != d.block_size ||
      s.head_dim != d.head_dim)
    return fail(PA_ERR_SHAPE, "source and destination caches differ in element type or block shape");
  if ((rc = check_tensor(block_mapping, "block_mapping", 2))) return rc;
  if (block_mapping->dtype != PA_I64) return fail(PA_ERR_DTYPE, "block_mapping must be int64");
  if (block_mapping->shape[1] != 2) return fail(PA_ERR_SHAPE, "block_mapping must be [num_pairs, 2]");
  const int64_t N = block_mapping->shape[0];
  if (N > 1 && block_mapping->stride[0] != 2) return fail(PA_ERR_LAYOUT, "block_mapping must be contiguous");
  if (block_mapping->stride[1] != 1) return fail(PA_ERR_LAYOUT, "block_mapping must be contiguous");
  const size_t e = elt_size(s.dtype);
  if ((s.block_size * s.head_dim * e) % 16 != 0)
    return fail(PA_ERR_UNSUPPORTED, "block tile must be a multiple of 16 bytes");
  if (N == 0) return PA_OK;
  DeviceState *ds;
  int dev;
  if ((rc = device_state(&ds, &dev))) return rc;
  void *p[5];
  const pa_tensor *ts[5] = {src_k, src_v, dst_k, dst_v, block_mapping};
  const char *names[5] = {"source key cache", "source value cache", "destination key cache",
                          "destination value cache", "block_mapping"};
  for (int i = 0; i < 5; ++i) {
    rc = host_allowed ? device_address(ts[i], names[i], dev, &p[i])
                      : check_device_memory(ts[i], names[i], dev);
    if (!host_allowed) p[i] = ts[i]->data;
    if (rc) return rc;
  }
  pa::CopyBlocksArgs a;
  a.src_key = static_cast<const char *>(p[0]);
  a.src_value = static_cast<const char *>(p[1]);
  a.dst_key = static_cast<char *>(p[2]);
  a.dst_value = static_cast<char *>(p[3]);
  a.src_blk = src_k->stride[0] * (int64_t)e;
  a.src_head = src_k->stride[1] * (int64_t)e;
  a.dst_blk = dst_k->stride[0] * (int64_t)e;
  a.dst_head = dst_k->stride[1] * (int64_t)e;
  a.tile_bytes = (int)(s.block_size * s.head_dim * e);
  a.pairs = static_cast<const int64_t *>(p[4]);
  a.num_pairs = N;
  a.num_kv_heads = s.num_kv_heads;
  a.src_blocks = s.num_blocks;
  a.dst_blocks = d.num_blocks;
  a.err = ds->err;
  cudaError_t err = pa::launch_copy_blocks(a, ds->num_sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? PA_OK : cuda_fail(err, host_allowed ? "swap_blocks launch" : "copy_blocks launch");
}

int write_fp8_impl(const pa_tensor *key, const pa_tensor *value, const pa_tensor *key_cache,
                   const pa_tensor *value_cache, const pa_tensor *slot_mapping,
                   const pa_tensor *k_scale, const pa_tensor *v_scale, void *stream,
                   CallMode mode = CallMode::kLaunch, pa::CacheWriteArgs *prepared = nullptr) {
  int rc;
  CacheShape cs;
  if ((rc = check_caches(key_cache, value_cache, &cs, true))) return rc;
  if (cs.dtype != PA_FP8_E4M3) return fail(PA_ERR_DTYPE, "pa_reshape_and_cache_fp8 needs fp8_e4m3 caches");
  if ((rc = check_tensor(key, "key", 3)) || (rc = check_tensor(value, "value", 3)) ||
      (rc = check_tensor(slot_mapping, "slot_mapping", 1)) ||
      (rc = check_tensor(k_scale, "k_scale", 1)) || (rc = check_tensor(v_scale, "v_scale", 1)))
    return rc;
  const int64_t T = key->shape[0];
  for (int i = 0; i < 3; ++i)
    if (value->shape[i] != key->shape[i]) return fail(PA_ERR_SHAPE, "key and value shapes differ");
  if (key->shape[1] != cs.num_kv_heads || key->shape[2] != cs.head_dim)
    return fail(PA_ERR_SHAPE, "key/value must be [num_tokens, num_kv_heads, head_dim] of the cache");
  if (slot_mapping->shape[0] != T) return fail(PA_ERR_SHAPE, "slot_mapping needs one slot per token");
  if (key->dtype != value->dtype || (key->dtype != PA_F32 && key->dtype != PA_BF16 && key->dtype != PA_F16))
    return fail(PA_ERR_DTYPE, "key/value must both be fp32, bf16 or fp16");
  if (slot_mapping->dtype != PA_I64) return fail(PA_ERR_DTYPE, "slot_mapping must be int64");
  if (k_scale->dtype != PA_F32 || v_scale->dtype != PA_F32)
    return fail(PA_ERR_DTYPE, "k_scale and v_scale must be fp32");
  if (k_scale->shape[0] != cs.num_kv_heads || v_scale->shape[0] != cs.num_kv_heads)
    return fail(PA_ERR_SHAPE, "k_scale and v_scale need one value per kv head");
  if ((k_scale->stride[0] != 1 || v_scale->stride[0] != 1) && cs.num_kv_heads > 1)
    return fail(PA_ERR_LAYOUT, "k_scale and v_scale must be contiguous");
  if (key->stride[2] != 1 || value->stride[2] != 1 || (slot_mapping->stride[0] != 1 && T > 1))
    return fail(PA_ERR_LAYOUT, "key/value need a contiguous head_dim and slot_mapping unit stride");
  if (!aligned16(key->data) || !aligned16(value->data) || !strides16(key, 2) || !strides16(value, 2))
    return fail(PA_ERR_LAYOUT, "key/value: data and token/head strides must be 16-byte aligned");
  if (cs.head_dim % 16 != 0) return fail(PA_ERR_UNSUPPORTED, "FP8 caches: head_dim must be a multiple of 16");
  if (T == 0 || mode == CallMode::kHostChecks) return PA_OK;
  DeviceState *ds;
  int dev;
  if ((rc = device_state(&ds, &dev))) return rc;
  if (mode != CallMode::kLaunchChecked &&
      ((rc = check_device_memory(key_cache, "key_cache", dev)) ||
       (rc = check_device_memory(value_cache, "value_cache", dev)) ||
       (rc = check_device_memory(key, "key", dev)) || (rc = check_device_memory(value, "value", dev)) ||
       (rc = check_device_memory(slot_mapping, "slot_mapping", dev)) ||
       (rc = check_device_memory(k_scale, "k_scale", dev)) ||
       (rc = check_device_memory(v_scale, "v_scale", dev))))
    return rc;
  const size_t se = elt_size(key->dtype);
  if (prepared) {
    // the same write done by the fused decode step (16-bit key/value rows, codes of head_dim
    // bytes per cache row)
    pa::CacheWriteArgs w;
    w.key = static_cast<const char *>(key->data);
    w.value = static_cast<const char *>(value->data);
    w.k_tok = key->stride[0] * (int64_t)se;
    w.k_head = key->stride[1] * (int64_t)se;
    w.v_tok = value->stride[0] * (int64_t)se;
    w.v_head = value->stride[1] * (int64_t)se;
    w.key_cache = static_cast<char *>(key_cache->data);
    w.value_cache = static_cast<char *>(value_cache->data);
    w.c_blk = key_cache->stride[0];
    w.c_head = key_cache->stride[1];
    w.row_bytes = cs.head_dim;
    w.slots = static_cast<const int64_t *>(slot_mapping->data);
    w.num_tokens = T;
    w.num_kv_heads = cs.num_kv_heads;
    w.block_size = cs.block_size;
    w.num_slots = cs.num_blocks * cs.block_size;
    w.err = ds->err;
    *prepared = w;
  }
  if (mode == CallMode::kAllChecks) return PA_OK;
  pa::CacheWriteFp8Args a;
  a.key = static_cast<const char *>(key->data);
  a.value = static_cast<const char *>(value->data);
  a.src_dtype = key->dtype;
  a.k_tok = key->stride[0] * (int64_t)se;
  a.k_head = key->stride[1] * (int64_t)se;
  a.v_tok = value->stride[0] * (int64_t)se;
  a.v_head = value->stride[1] * (int64_t)se;
  a.key_cache = static_cast<unsigned char *>(key_cache->data);
  a.value_cache = static_cast<unsigned char *>(value_cache->data);
  a.c_blk = key_cache->stride[0];
  a.c_head = key_cache->stride[1];
  a.head_dim = cs.head_dim;
  a.slots = static_cast<const int64_t *>(slot_mapping->data);
  a.num_tokens = T;
  a.num_kv_heads = cs.num_kv_heads;
  a.block_size = cs.block_size;
  a.num_slots = cs.num_blocks * cs.block_size;
  a.k_scale = static_cast<const float *>(k_scale->data);
  a.v_scale = static_cast<const float *>(v_scale->data);
  a.err = ds->err;
  cudaError_t err = pa::launch_reshape_and_cache_fp8(a, ds->num_sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? PA_OK : cuda_fail(err, "reshape_and_cache_fp8 launch");
}

}  // namespace

extern "C" {

int pa_prefill(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
               const pa_tensor *value_cache, const pa_tensor *block_tables,
               const pa_tensor *context_lens, const pa_tensor *query_start, float scale,
               int32_t block_size, int32_t num_kv_heads, void *stream) {
  int rc;
  CacheShape cs;
  if ((rc = check_caches(key_cache, value_cache, &cs))) return rc;
  if ((rc = check_tensor(query, "query", 3)) || (rc = check_tensor(out, "out", 3)) ||
      (rc = check_tensor(block_tables, "block_tables", 2)) ||
      (rc = check_tensor(context_lens, "context_lens", 1)) ||
      (rc = check_tensor(query_start, "query_start", 1)))
    return rc;
  if (block_size != cs.block_size)
    return fail(PA_ERR_SHAPE, "block_size %d does not match the cache's %d", block_size, cs.block_size);
  if (num_kv_heads != cs.num_kv_heads)
    return fail(PA_ERR_SHAPE, "num_kv_heads %d does not match the cache's %d", num_kv_heads, cs.num_kv_heads);
  const int64_t S = context_lens->shape[0];
  const int64_t T = query->shape[0];
  const int64_t Hq = query->shape[1];
  const int D = cs.head_dim;
  if (query->shape[2] != D) return fail(PA_ERR_SHAPE, "query head_dim %lld != cache head_dim %d", (long long)query->shape[2], D);
  if (out->shape[0] != T || out->shape[1] != Hq || out->shape[2] != D)
    return fail(PA_ERR_SHAPE, "out must be [num_tokens, num_heads, head_dim] like query");
  if (block_tables->shape[0] != S || query_start->shape[0] != S + 1)
    return fail(PA_ERR_SHAPE, "block_tables needs one row and query_start S + 1 entries for S sequences");
  if (cs.dtype != PA_BF16 && cs.dtype != PA_F16)
    return fail(PA_ERR_UNSUPPORTED, "prefill is built for bf16 and fp16 caches");
  if (query->dtype != cs.dtype) return fail(PA_ERR_DTYPE, "query must have the caches' element type");
  if (out->dtype != PA_F32 && out->dtype != cs.dtype)
    return fail(PA_ERR_DTYPE, "out must be fp32 or the caches' element type");
  if (block_tables->dtype != PA_I32 || context_lens->dtype != PA_I32 || query_start->dtype != PA_I32)
    return fail(PA_ERR_DTYPE, "block_tables, context_lens and query_start must be int32");
  if (Hq <= 0 && T > 0) return fail(PA_ERR_SHAPE, "num_heads must be positive");
  if (Hq % num_kv_heads != 0) return fail(PA_ERR_SHAPE, "num_heads %lld is not a multiple of num_kv_heads %d", (long long)Hq, num_kv_heads);
  const int G = (int)(Hq / num_kv_heads);
  if (D != 64 && D != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d (built: 64, 128)", D);
  if (block_size != 8 && block_size != 16 && block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "block_size %d (built: 8, 16, 32)", block_size);
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per kv head %d (built: 1, 2, 4, 8)", G);
  if (query->stride[2] != 1 || out->stride[2] != 1)
    return fail(PA_ERR_LAYOUT, "query and out need a contiguous head_dim");
  if (!aligned16(query->data) || !strides16(query, 2) || !aligned16(out->data) || !strides16(out, 2))
    return fail(PA_ERR_LAYOUT, "query/out: data and token/head strides must be 16-byte aligned");
  if (block_tables->stride[1] != 1 && block_tables->shape[1] > 1)
    return fail(PA_ERR_LAYOUT, "block_tables rows must be contiguous");
  if ((context_lens->stride[0] != 1 && S > 1) || query_start->stride[0] != 1)
    return fail(PA_ERR_LAYOUT, "context_lens and query_start must be contiguous");
  if (S > 0x7fffffff || T > 0x7fffffff || block_tables->shape[1] * block_size > 0x7fffffff)
    return fail(PA_ERR_SHAPE, "too many sequences or tokens, or too long a block table");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  if (S == 0 || T == 0) return PA_OK;
  DeviceState *ds;
  int dev;
  if ((rc = device_state(&ds, &dev))) return rc;
  if ((rc = check_device_memory(key_cache, "key_cache", dev)) ||
      (rc = check_device_memory(value_cache, "value_cache", dev)) ||
      (rc = check_device_memory(query, "query", dev)) || (rc = check_device_memory(out, "out", dev)) ||
      (rc = check_device_memory(block_tables, "block_tables", dev)) ||
      (rc = check_device_memory(context_lens, "context_lens", dev)) ||
      (rc = check_device_memory(query_start, "query_start", dev)))
    return rc;
  pa::PrefillKernel k;
  const bool got = cs.dtype == PA_BF16 ? pa::prefill_kernel_bf16(D, block_size, G, &k)
                                       : pa::prefill_kernel_f16(D, block_size, G, &k);
  if (!got)
    return fail(PA_ERR_CUDA, "could not prepare the prefill kernel: %s", cudaGetErrorString(cudaGetLastError()));
  pa::PrefillMaps maps;
  // one box per (block, kv head) tile when the caches allow the grouped view, else 8-row boxes
  const bool grouped = grouped_view_ok(key_cache) && grouped_view_ok(value_cache);
  const int rows = grouped ? 0 : k.tma_rows;
  if ((rc = cache_map(key_cache, rows, &maps.k)) || (rc = cache_map(value_cache, rows, &maps.v)) ||
      (rc = query_map(query, G, &maps.q)))
    return rc;
  // enough CTAs for every tile of any split of T tokens among S sequences, at most one wave
  const int64_t tiles = ((T + k.tokens_per_tile - 1) / k.tokens_per_tile + S) * num_kv_heads;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.kernel, k.threads_per_cta,
                                                    k.smem_bytes) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t wave = (int64_t)per_sm * ds->num_sms;
  const int ctas = (int)(tiles < wave ? tiles : wave);
  pa::PrefillArgs a = {};
  a.out = out->data;
  a.out_dtype = out->dtype;
  a.out_t = out->stride[0];
  a.out_h = out->stride[1];
  a.query = query->data;
  a.q_t = query->stride[0];
  a.q_h = query->stride[1];
  a.block_tables = static_cast<const int32_t *>(block_tables->data);
  a.bt_s = block_tables->stride[0];
  a.context_lens = static_cast<const int32_t *>(context_lens->data);
  a.query_start = static_cast<const int32_t *>(query_start->data);
  a.num_seqs = (int)S;
  a.num_kv_heads = num_kv_heads;
  a.max_blocks = (int)block_tables->shape[1];
  a.num_blocks = cs.num_blocks;
  a.num_tokens = T;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.err = ds->err;
  a.wait_cycles = test_hooks().wait_cycles;
  a.grouped_maps = grouped ? 1 : 0;
  cudaError_t e = k.launch(a, &maps, ctas, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "prefill launch");
}

int pa_reshape_and_cache_fp8(const pa_tensor *key, const pa_tensor *value,
                             const pa_tensor *key_cache, const pa_tensor *value_cache,
                             const pa_tensor *slot_mapping, const pa_tensor *k_scale,
                             const pa_tensor *v_scale, void *stream) {
  return write_fp8_impl(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale, stream);
}

int pa_decode_fp8(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                  const pa_tensor *value_cache, const pa_tensor *block_tables,
                  const pa_tensor *context_lens, const pa_tensor *k_scale,
                  const pa_tensor *v_scale, float scale, int32_t block_size, int32_t num_kv_heads,
                  int32_t num_workers, uint32_t flags, void *workspace, size_t workspace_bytes,
                  void *stream) {
  if (!k_scale || !v_scale) return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale are required");
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, num_workers, flags, workspace, workspace_bytes,
                     workspace == nullptr, stream, CallMode::kLaunch, k_scale, v_scale);
}

int pa_reshape_and_cache(const pa_tensor *key, const pa_tensor *value, const pa_tensor *key_cache,
                         const pa_tensor *value_cache, const pa_tensor *slot_mapping, void *stream) {
  return write_impl(key, value, key_cache, value_cache, slot_mapping, stream, CallMode::kLaunch);
}

int pa_decode_step_fp8(const pa_tensor *key, const pa_tensor *value, const pa_tensor *key_cache,
                       const pa_tensor *value_cache, const pa_tensor *slot_mapping,
                       const pa_tensor *k_scale, const pa_tensor *v_scale, const pa_tensor *out,
                       const pa_tensor *query, const pa_tensor *block_tables,
                       const pa_tensor *context_lens, float scale, int32_t block_size,
                       int32_t num_kv_heads, void *workspace, size_t workspace_bytes,
                       void *stream) {
  if (!k_scale || !v_scale) return fail(PA_ERR_INVALID_ARG, "k_scale and v_scale are required");
  const bool lib_ws = workspace == nullptr;
  int rc;
  // One new token per sequence, in the query's 16-bit type: one kernel, which quantises the
  // token into the caches and into its tiles as position L-1.  Otherwise the write kernel, then
  // the decode launched to overlap it.
  const bool fused = key && query && context_lens && key->ndim == 3 && context_lens->ndim == 1 &&
                     key->shape[0] == context_lens->shape[0] && key->dtype == query->dtype;
  pa::CacheWriteArgs w;
  for (CallMode m : {CallMode::kHostChecks, CallMode::kAllChecks})
    if ((rc = write_fp8_impl(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale,
                             stream, m, fused ? &w : nullptr)) ||
        (rc = decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                          block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                          workspace_bytes, lib_ws, stream, m, k_scale, v_scale)))
      return rc;
  if (fused) {
    if (key->shape[0] == 0) return PA_OK;
    return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                       block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                       workspace_bytes, lib_ws, stream, CallMode::kLaunchChecked, k_scale,
                       v_scale, nullptr, nullptr, &w);
  }
  if ((rc = write_fp8_impl(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale,
                           stream, CallMode::kLaunchChecked)))
    return rc;
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                     workspace_bytes, lib_ws, stream, CallMode::kLaunchChecked, k_scale, v_scale);
}

int pa_decode_step(const pa_tensor *key, const pa_tensor *value, const pa_tensor *key_cache,
                   const pa_tensor *value_cache, const pa_tensor *slot_mapping,
                   const pa_tensor *out, const pa_tensor *query, const pa_tensor *block_tables,
                   const pa_tensor *context_lens, float scale, int32_t block_size,
                   int32_t num_kv_heads, void *workspace, size_t workspace_bytes, void *stream) {
  const bool lib_ws = workspace == nullptr;
  int rc;
  // One new token per sequence in 16-bit caches: one kernel for the whole step, which writes
  // the caches and decodes with token s as sequence s's position L-1 (read from key / value,
  // so the decode never waits for the write).  Otherwise: the write kernel, then the decode.
  const bool fused = key && query && context_lens && key_cache && key->ndim == 3 &&
                     context_lens->ndim == 1 && key->shape[0] == context_lens->shape[0] &&
                     (key_cache->dtype == PA_BF16 || key_cache->dtype == PA_F16);
  if (fused) {
    pa::CacheWriteArgs w;
    for (CallMode m : {CallMode::kHostChecks, CallMode::kAllChecks})
      if ((rc = write_impl(key, value, key_cache, value_cache, slot_mapping, stream, m, &w)) ||
          (rc = decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                            block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                            workspace_bytes, lib_ws, stream, m)))
        return rc;
    if (key->shape[0] > 0)
      return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                         block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                         workspace_bytes, lib_ws, stream, CallMode::kLaunchChecked, nullptr,
                         nullptr, nullptr, nullptr, &w);
    return PA_OK;
  }
  // both halves are checked (host-side checks of both first) before either is launched
  for (CallMode m : {CallMode::kHostChecks, CallMode::kAllChecks})
    if ((rc = write_impl(key, value, key_cache, value_cache, slot_mapping, stream, m)) ||
        (rc = decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                          block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                          workspace_bytes, lib_ws, stream, m)))
      return rc;
  if ((rc = write_impl(key, value, key_cache, value_cache, slot_mapping, stream,
                      CallMode::kLaunchChecked)))
    return rc;
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, 0, PA_DECODE_OVERLAP_PREVIOUS, workspace,
                     workspace_bytes, lib_ws, stream, CallMode::kLaunchChecked);
}

int pa_copy_blocks(const pa_tensor *key_cache, const pa_tensor *value_cache,
                   const pa_tensor *block_mapping, void *stream) {
  return copy_blocks_impl(key_cache, value_cache, key_cache, value_cache, block_mapping, false,
                          stream);
}

int pa_swap_blocks(const pa_tensor *src_key_cache, const pa_tensor *src_value_cache,
                   const pa_tensor *dst_key_cache, const pa_tensor *dst_value_cache,
                   const pa_tensor *block_mapping, void *stream) {
  return copy_blocks_impl(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache,
                          block_mapping, true, stream);
}

int pa_decode(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
              const pa_tensor *value_cache, const pa_tensor *block_tables,
              const pa_tensor *context_lens, float scale, int32_t block_size,
              int32_t num_kv_heads, void *stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, 0, 0u, nullptr, 0, true, stream);
}

int pa_decode_ex(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                 const pa_tensor *value_cache, const pa_tensor *block_tables,
                 const pa_tensor *context_lens, float scale, int32_t block_size,
                 int32_t num_kv_heads, int32_t num_workers, uint32_t flags, void *workspace,
                 size_t workspace_bytes, void *stream) {
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, num_workers, flags, workspace, workspace_bytes,
                     false, stream);
}

int pa_decode_shared_prefix(const pa_tensor *out, const pa_tensor *query, const pa_tensor *key_cache,
                            const pa_tensor *value_cache, const pa_tensor *block_tables,
                            const pa_tensor *context_lens, const pa_tensor *group_start,
                            const pa_tensor *prefix_lens, float scale, int32_t block_size,
                            int32_t num_kv_heads, void *workspace, size_t workspace_bytes,
                            void *stream) {
  if (!group_start) return fail(PA_ERR_INVALID_ARG, "group_start is required");
  return decode_impl(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                     block_size, num_kv_heads, 0, 0u, workspace, workspace_bytes,
                     workspace == nullptr, stream, CallMode::kLaunch, nullptr, nullptr,
                     group_start, prefix_lens);
}

size_t pa_decode_shared_prefix_workspace_bytes(int64_t num_seqs, int32_t num_heads,
                                               int32_t num_kv_heads, int32_t head_dim,
                                               int64_t max_blocks_per_seq, int32_t block_size) {
  if (max_blocks_per_seq < 0 || block_size <= 0) return 0;
  const size_t base = pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, 0);
  if (base == 0) return 0;
  return prefix_layout(base, num_seqs, num_heads, head_dim, max_blocks_per_seq, block_size).total;
}

size_t pa_decode_workspace_bytes(int64_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t num_workers) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_workers < 0 ||
      num_heads % num_kv_heads != 0)
    return 0;
  int W = num_workers;
  if (W == 0) {
    DeviceState *ds;
    if (device_state(&ds, nullptr) != PA_OK) return 0;
    W = ds->num_sms * 16;  // at most 4 CTAs of 4 warps per SM for any built configuration
  }
  return ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, W).total;
}

int32_t pa_decode_default_workers(int32_t dtype, int32_t head_dim, int32_t block_size,
                                  int32_t group_size) {
  DeviceState *ds;
  if (device_state(&ds, nullptr) != PA_OK) return 0;
  pa::DecodeKernel k;
  if (!get_kernel(dtype, head_dim, block_size, group_size, dtype != PA_F32, &k)) return 0;
  return default_workers(k, ds->num_sms);
}

int pa_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (!workspace && workspace_bytes) return fail(PA_ERR_INVALID_ARG, "NULL workspace");
  if (!workspace_bytes) return PA_OK;
  cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
  std::lock_guard<std::mutex> lock(g_mu);
  clean_record(workspace).clean = workspace_bytes;
  return PA_OK;
}

int pa_release_workspaces(void) {
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(g_mu);
  for (size_t d = 0; d < g_devices.size(); ++d) {
    if (!g_devices[d].ws) continue;
    cudaSetDevice((int)d);
    cudaDeviceSynchronize();
    cudaFree(g_devices[d].ws);
    for (auto &r : g_clean)
      if (r.ws == g_devices[d].ws) r.clean = 0;
    g_devices[d].ws = nullptr;
    g_devices[d].ws_bytes = 0;
  }
  cudaSetDevice(cur);
  return PA_OK;
}

const char *pa_last_error(void) { return g_last_error.c_str(); }

int pa_set_decode_timeline(void *buf, size_t bytes) {
  if (buf && ((uintptr_t)buf & 7u) != 0) return fail(PA_ERR_LAYOUT, "timeline buffer must be 8-byte aligned");
  std::lock_guard<std::mutex> lock(g_mu);
  g_timeline = static_cast<unsigned long long *>(buf);
  g_timeline_warps = buf ? (long long)(bytes / (pa::kTimelineWords * 8)) : 0;
  return PA_OK;
}

int pa_get_device_error(void *stream, uint32_t *flags, int32_t clear) {
  if (!flags) return fail(PA_ERR_INVALID_ARG, "flags is NULL");
  DeviceState *ds;
  int rc = device_state(&ds, nullptr);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, ds->err, sizeof(host), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  *flags = host;
  if (host & PA_DEVERR_TIMEOUT) {
    // An abandoned decode may have left merge counters partly counted in whichever workspace
    // it used: every workspace this library has seen (its own, the callers', the static
    // scratch of pa_decode_noalloc) gets its counters zeroed again before its next use.
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto &r : g_clean) r.clean = 0;
  }
  if (clear) {
    e = cudaMemsetAsync(ds->err, 0, sizeof(unsigned int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  }
  return PA_OK;
}

int32_t pa_version(void) { return PA_VERSION; }

}  // extern "C"
