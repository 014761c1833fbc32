// C ABI of the paged GQA/MQA decode-attention library (declared in include/gqa_decode.h).
//
// Host responsibilities: argument validation (nothing is launched on a bad argument),
// the per-device workspace (error word, split counters, split partials), TMA tensor
// maps over the page pools, and kernel launches.  No call synchronises the stream
// except gqa_check_device_error.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "gqa_decode.h"
#include "internal.cuh"

namespace {

thread_local char g_err_msg[512] = "no error";
std::atomic<int> g_num_workers{0};
std::atomic<int64_t> g_wait_limit_ns{1000000000LL};
std::atomic<int> g_arm_without_copy{0};
std::atomic<uint64_t> g_launches{0};

gqa_status fail(gqa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err_msg, sizeof(g_err_msg), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace

gqa_status gqa::set_error(gqa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err_msg, sizeof(g_err_msg), fmt, ap);
  va_end(ap);
  return s;
}

namespace {

gqa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(GQA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------ per-device state
struct DeviceState {
  int sms = 0;
  uint32_t* err = nullptr;
  int32_t* counters = nullptr;
  size_t counters_cap = 0;  // entries
  float* part_o = nullptr;
  float* part_ml = nullptr;
  size_t part_o_cap = 0;    // floats
  size_t part_ml_cap = 0;   // floats
};

std::mutex g_mu;
std::unordered_map<int, DeviceState> g_states;

// The state of the current device if a call has set it up already (never creates it).
DeviceState* existing_state(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_states.find(dev);
  return (it == g_states.end() || it->second.err == nullptr) ? nullptr : &it->second;
}

gqa_status get_state(DeviceState** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_states[dev];
  if (s.err == nullptr) {
    e = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaMalloc(&s.err, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(error word)");
    e = cudaMemset(s.err, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error word)");
  }
  *out = &s;
  *dev_out = dev;
  return GQA_OK;
}

// Grow-only decode workspace.  Counters must be zero between launches: they are
// zeroed when allocated and every launch leaves them zero.
gqa_status ensure_workspace(DeviceState& s, size_t counters, size_t part_o_floats,
                            size_t part_ml_floats, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  cudaError_t e;
  if (counters > s.counters_cap) {
    if (s.counters) cudaFree(s.counters);
    s.counters = nullptr;
    s.counters_cap = 0;
    size_t n = counters < 4096 ? 4096 : counters;
    e = cudaMalloc(&s.counters, n * sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(split counters)");
    e = cudaMemsetAsync(s.counters, 0, n * sizeof(int32_t), stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(split counters)");
    s.counters_cap = n;
  }
  if (part_o_floats > s.part_o_cap) {
    if (s.part_o) cudaFree(s.part_o);
    s.part_o = nullptr;
    s.part_o_cap = 0;
    e = cudaMalloc(&s.part_o, part_o_floats * sizeof(float));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(split partials)");
    s.part_o_cap = part_o_floats;
  }
  if (part_ml_floats > s.part_ml_cap) {
    if (s.part_ml) cudaFree(s.part_ml);
    s.part_ml = nullptr;
    s.part_ml_cap = 0;
    e = cudaMalloc(&s.part_ml, part_ml_floats * sizeof(float));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(split partials)");
    s.part_ml_cap = part_ml_floats;
  }
  return GQA_OK;
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// The pool [num_pages, Hk, ps, D] viewed as a 3-D bf16 tensor: 64 columns (128 bytes)
// x P*Hk*ps rows x D/64 column groups (stride 128 bytes).  One box is 64 columns x 16
// rows (one sub-chunk) x all D/64 groups, 128-byte swizzle; in shared memory it lands
// as D/64 consecutive [16, 64] tiles.
struct MapKey {
  const void* ptr;
  const void* ptr2;  // the second pool of a paired map (make_map_pair), else nullptr
  int64_t rows;
  int d;
  int dev;
  int box_rows;
  int box_groups;
  int codes;  // 1: an e4m3 pool (make_map_codes), 0: bf16
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && ptr2 == o.ptr2 && rows == o.rows && d == o.d && dev == o.dev &&
           box_rows == o.box_rows && box_groups == o.box_groups && codes == o.codes;
  }
};

// A [rows, d] bf16 matrix viewed as a 3-D tensor: 64 columns (128 bytes) x rows x d/64
// column groups (stride 128 bytes).  One box is 64 columns x box_rows rows x box_groups
// groups, 128-byte swizzle; it lands as box_groups consecutive [box_rows, 64] tiles.
// Used for the page pools ([P * Hk * ps, D]) and for q ([B * H, D]).
gqa_status make_map(CUtensorMap* m, const void* base, int64_t rows, int d, int dev, int box_rows,
                    int box_groups) {
  static thread_local MapKey keys[8];
  static thread_local CUtensorMap maps[8];
  static thread_local int next = 0;
  MapKey k{base, nullptr, rows, d, dev, box_rows, box_groups, 0};
  for (int i = 0; i < 8; ++i)
    if (keys[i] == k) {
      *m = maps[i];
      return GQA_OK;
    }
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(d / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_groups)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  keys[next] = k;
  maps[next] = *m;
  next = (next + 1) % 8;
  return GQA_OK;
}

// An e4m3 pool [P * Hk * ps, D] (one byte per element) viewed as 128-byte rows: a 2-D
// uint8 tensor of 128 columns x rows * D / 128 rows.  One box is box_rows of those rows,
// 128-byte swizzle (16 tokens of codes are 16 * D / 128 rows).
gqa_status make_map_codes(CUtensorMap* m, const void* base, int64_t rows, int d, int dev, int box_rows) {
  static thread_local MapKey keys[4];
  static thread_local CUtensorMap maps[4];
  static thread_local int next = 0;
  MapKey k{base, nullptr, rows, d, dev, box_rows, 1, 1};
  for (int i = 0; i < 4; ++i)
    if (keys[i] == k) {
      *m = maps[i];
      return GQA_OK;
    }
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows * d / 128)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled (e4m3 pool) failed (%d)", (int)r);
  keys[next] = k;
  maps[next] = *m;
  next = (next + 1) % 4;
  return GQA_OK;
}

// The K and V e4m3 pools ([P * Hk * ps, D] codes each) as one tensor of 128-byte rows
// with an outer coordinate of extent 2 whose stride is the distance between the pools,
// based at the lower one: one copy then brings a 16-token sub-chunk of K and of V,
// landing as the lower pool's tile followed by the other's.  The copy touches only rows
// of the two pools.  Returns 0 when the pools cannot be paired (the same pool, or a
// distance the tensor map cannot express: not a multiple of 16 bytes, or 2^40 bytes or
// more), else 1 when K is the lower pool and 2 when V is; *st reports an encoding
// failure.  (Pairing the bf16 pools as well measured mixed: 1 % faster on the long-context
// batch, 1-2 % slower on the 32-sequence GQA batch; they keep separate maps.)
int make_map_pair(CUtensorMap* m, const void* k_pages, const void* v_pages, int64_t rows, int d, int dev,
                  gqa_status* st) {
  *st = GQA_OK;
  const uintptr_t ka = reinterpret_cast<uintptr_t>(k_pages), va = reinterpret_cast<uintptr_t>(v_pages);
  if (ka == va) return 0;
  const uint64_t dist = ka < va ? va - ka : ka - va;
  if (dist % 16 != 0 || dist >= (uint64_t{1} << 40)) return 0;
  const int order = ka < va ? 1 : 2;
  const void* lo = ka < va ? k_pages : v_pages;
  const void* hi = ka < va ? v_pages : k_pages;
  static thread_local MapKey keys[4];
  static thread_local CUtensorMap maps[4];
  static thread_local int next = 0;
  MapKey key{lo, hi, rows, d, dev, gqa::kChunk, 1, 1};
  for (int i = 0; i < 4; ++i)
    if (keys[i] == key) {
      *m = maps[i];
      return order;
    }
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *st = fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    return 0;
  }
  // 128 columns x 128-byte rows of codes x the two pools
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows * d / 128), 2};
  cuuint64_t strides[2] = {128, dist};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(gqa::kChunk * d / 128), 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(lo), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return 0;  // not expressible here: separate maps instead
  keys[next] = key;
  maps[next] = *m;
  next = (next + 1) % 4;
  return order;
}

// Query rows of several tokens per sequence for the tcgen05 kernel, as a 5-D view of
// q [B, Q, Hk * G, D]: (64 columns, head in group, token, column group, b * Q * Hk + kvh).
// The last coordinate's stride is G * D elements: (b * Q * Hk + kvh) * G * D is the first
// element of kv head kvh's group for token 0 of sequence b.  One box = the G x Q rows of a
// (sequence, kv head) and one column group, landing as rows (token, head) of the tile.
gqa_status make_qmap_multi(CUtensorMap* m, const void* base, int B, int Q, int Hk, int G, int d) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(Q), static_cast<cuuint64_t>(d / 64),
                        static_cast<cuuint64_t>(static_cast<int64_t>(B - 1) * Q * Hk + Hk)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Hk) * G * d * 2, 128,
                           static_cast<cuuint64_t>(G) * d * 2};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(Q), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled (5-D query map) failed (%d)", (int)r);
  return GQA_OK;
}

// Tensor maps of one decode launch and the launch itself (both kernels).
cudaError_t launch_with_maps(gqa::DecodeParams p, const gqa::DecodePlan& plan,
                             const void* q, const void* k_pages, const void* v_pages, int64_t rows,
                             int dev, int grid, cudaStream_t strm, bool overlap, gqa_status* st) {
  CUtensorMap tk, tv, tq;
  gqa::divisor_magic(static_cast<uint32_t>(p.page_size), &p.ps_magic, &p.ps_shift);
  const int hd = p.head_dim;
  if (plan.tensor_cores) {
    const int br = gqa::tc_box_rows(p.page_size);
    const int bg = br == 64 ? hd / 64 : 1;  // a 64-row box carries every column group
    if (p.k_scales != nullptr) {  // e4m3 codes: br tokens are br * D / 128 rows of 128 bytes
      *st = make_map_codes(&tk, k_pages, rows, hd, dev, br * hd / 128);
      if (*st == GQA_OK) *st = make_map_codes(&tv, v_pages, rows, hd, dev, br * hd / 128);
    } else {
      *st = make_map(&tk, k_pages, rows, hd, dev, br, bg);
      if (*st == GQA_OK) *st = make_map(&tv, v_pages, rows, hd, dev, br, bg);
    }
    if (*st == GQA_OK)
      *st = p.q_len > 1
                ? make_qmap_multi(&tq, q, p.num_seqs, p.q_len, p.num_kv_heads, p.group, hd)
                : make_map(&tq, q, static_cast<int64_t>(p.num_seqs) * p.num_heads, hd, dev, 128, hd / 64);
    if (*st != GQA_OK) return cudaSuccess;
    return gqa::launch_decode_tc(p, tk, tv, tq, grid, strm, overlap);
  }
  // e4m3 codes: one copy per sub-chunk for K and V when the pools can share a map
  // (41.9 against 43.2 us on the GQA batch, 216.6 against 221 on the long-context one)
  p.kv_pair = p.k_scales != nullptr ? make_map_pair(&tk, k_pages, v_pages, rows, hd, dev, st) : 0;
  if (*st != GQA_OK) return cudaSuccess;
  if (p.kv_pair != 0) {
    tv = tk;  // unused by the kernel
  } else if (p.k_scales != nullptr) {  // e4m3 codes: a 16-token sub-chunk is 16 * D / 128 rows of 128 bytes
    *st = make_map_codes(&tk, k_pages, rows, hd, dev, gqa::kChunk * hd / 128);
    if (*st == GQA_OK) *st = make_map_codes(&tv, v_pages, rows, hd, dev, gqa::kChunk * hd / 128);
  } else {
    *st = make_map(&tk, k_pages, rows, hd, dev, gqa::kChunk, hd / 64);
    if (*st == GQA_OK) *st = make_map(&tv, v_pages, rows, hd, dev, gqa::kChunk, hd / 64);
  }
  if (*st != GQA_OK) return cudaSuccess;
  return gqa::launch_decode(p, plan, tk, tv, grid, strm, overlap);
}

}  // namespace

// ------------------------------------------------------------------ allocation-free decode
// Scratch of gqa_paged_decode_attn_noalloc: a fixed array in the library's device
// image, present on every GPU that loads the library until the process exits, so the
// call never has to allocate.  Layout per call: the device error word (first 256
// bytes), one arrival counter per segment, then the split partials (reference max and
// sum, then unnormalised O) of two slots per worker.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;  // 16 MiB
constexpr size_t kNoAllocHeaderBytes = 256;
constexpr size_t kNoAllocMaxSegments = 16384;             // num_seqs * num_kv_heads * head tiles
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
std::unordered_map<int, std::pair<unsigned char*, int>> g_noalloc_dev;  // device -> (address, SMs)

// Host code only holds a stand-in for g_noalloc_scratch; its device address is looked
// up once per device, with that device current.
gqa_status noalloc_scratch(int dev, unsigned char** ptr, int* sms) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  auto it = g_noalloc_dev.find(dev);
  if (it == g_noalloc_dev.end()) {
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(allocation-free scratch)");
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    // The error word starts at zero; after this it is cleared only when
    // gqa_check_device_error reads it, so errors of any call stay visible until then.
    e = cudaMemset(addr, 0, kNoAllocHeaderBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(allocation-free error word)");
    it = g_noalloc_dev.emplace(dev, std::make_pair(static_cast<unsigned char*>(addr), n)).first;
  }
  *ptr = it->second.first;
  *sms = it->second.second;
  return GQA_OK;
}

// The scratch address of a device whose allocation-free set-up has run, else nullptr.
unsigned char* noalloc_scratch_if_set_up(int dev) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  auto it = g_noalloc_dev.find(dev);
  return it == g_noalloc_dev.end() ? nullptr : it->second.first;
}

size_t align256(size_t x) { return (x + 255) & ~size_t{255}; }

gqa_status decode_impl(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* block_table, const int32_t* seq_lens, void* out,
                       int num_seqs, int num_heads, int num_kv_heads, int head_dim, int page_size,
                       float scale, int max_blocks_per_seq, int num_pages, void* stream,
                       bool overlap_previous, int q_len = 1, const float* k_scales = nullptr,
                       const float* v_scales = nullptr) {
  const bool fp8 = k_scales != nullptr || v_scales != nullptr;
  if (num_seqs < 0) return fail(GQA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_seqs > 65536) return fail(GQA_ERR_UNSUPPORTED, "num_seqs > 65536");
  if (q_len < 1) return fail(GQA_ERR_INVALID_ARG, "q_len %d < 1", q_len);
  if (num_heads < 1 || num_kv_heads < 1 || head_dim < 1 || page_size < 1 ||
      max_blocks_per_seq < 1 || num_pages < 1)
    return fail(GQA_ERR_INVALID_ARG, "sizes must be positive");
  if (num_heads % num_kv_heads != 0)
    return fail(GQA_ERR_INVALID_ARG, "num_heads (%d) is not a multiple of num_kv_heads (%d)",
                num_heads, num_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(GQA_ERR_UNSUPPORTED, "head_dim %d not built (64, 128)", head_dim);
  if (page_size % gqa::kChunk != 0 || page_size > 256)
    return fail(GQA_ERR_UNSUPPORTED, "page_size %d not built (multiple of 16, <= 256)", page_size);
  if (!std::isfinite(scale)) return fail(GQA_ERR_INVALID_ARG, "scale is not finite");
  const int64_t rows = static_cast<int64_t>(num_pages) * num_kv_heads * page_size;
  if (rows >= (int64_t{1} << 31))
    return fail(GQA_ERR_UNSUPPORTED, "num_pages * num_kv_heads * page_size exceeds 2^31");
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size >= (int64_t{1} << 31))
    return fail(GQA_ERR_UNSUPPORTED, "max_blocks_per_seq * page_size exceeds 2^31");
  // Several query tokens: each kv head's rows are its group for every token, read with
  // one pass over its K/V (one segment of at most 128 rows).
  if (q_len > 1 && static_cast<int64_t>(num_heads / num_kv_heads) * q_len > 128)
    return fail(GQA_ERR_UNSUPPORTED, "q_len %d x %d query heads per kv head exceeds 128", q_len,
                num_heads / num_kv_heads);
  if (num_seqs == 0) return GQA_OK;
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out)
    return fail(GQA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(k_pages, 16) || !aligned(v_pages, 16))
    return fail(GQA_ERR_INVALID_ARG, "k_pages / v_pages must be 16-byte aligned");
  if (!aligned(q, 16) || !aligned(out, 8))
    return fail(GQA_ERR_INVALID_ARG, "q must be 16-byte and out 8-byte aligned");
  if (fp8) {
    if (k_scales == nullptr || v_scales == nullptr)
      return fail(GQA_ERR_INVALID_ARG, "k_scales and v_scales are both required");
    if (!aligned(k_scales, 4) || !aligned(v_scales, 4))
      return fail(GQA_ERR_INVALID_ARG, "k_scales / v_scales must be 4-byte aligned");
    if (q_len != 1) return fail(GQA_ERR_UNSUPPORTED, "the 8-bit cache serves one query token per sequence");
  }

  DeviceState* st;
  int dev;
  gqa_status s = get_state(&st, &dev);
  if (s != GQA_OK) return s;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);

  const int group = num_heads / num_kv_heads;
  const gqa::DecodePlan plan = gqa::plan_decode(head_dim, group * q_len, q_len > 1, fp8);
  // Upper bound on the block count (seq_lens are device data).
  const int64_t blocks_per_seq =
      (static_cast<int64_t>(max_blocks_per_seq) * page_size + gqa::kBlock - 1) / gqa::kBlock;
  const int64_t max_blocks = static_cast<int64_t>(num_seqs) * num_kv_heads * plan.n_ht * blocks_per_seq;
  int64_t workers = static_cast<int64_t>(st->sms) * plan.ctas_per_sm;
  const int forced = g_num_workers.load();
  if (forced > 0) workers = forced;
  if (workers > max_blocks) workers = max_blocks;
  if (workers < 1) workers = 1;
  const int grid = static_cast<int>(workers);

  const size_t segments = static_cast<size_t>(num_seqs) * num_kv_heads * plan.n_ht;
  const size_t slots = static_cast<size_t>(2 * workers);
  s = ensure_workspace(*st, segments, slots * plan.heads_per_seg * head_dim,
                       slots * plan.heads_per_seg * 2, strm);
  if (s != GQA_OK) return s;


  gqa::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.part_o = st->part_o;
  p.part_ml = st->part_ml;
  p.counters = st->counters;
  p.err = st->err;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.n_ht = plan.n_ht;
  p.heads_per_seg = plan.heads_per_seg;
  p.page_size = page_size;
  p.max_blocks = max_blocks_per_seq;
  p.num_pages = num_pages;
  p.head_dim = head_dim;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_workers = static_cast<int>(workers);
  p.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns.load());
  p.arm_without_copy = g_arm_without_copy.load();
  p.q_len = q_len;
  cudaError_t e = launch_with_maps(p, plan, q, k_pages, v_pages, rows, dev, grid, strm,
                                   overlap_previous, &s);
  if (s != GQA_OK) return s;
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  g_launches.fetch_add(plan.tensor_cores && grid > 1 ? 2 : 1);
  return GQA_OK;
}

}  // namespace

namespace {

gqa_status append_impl(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                       const int32_t* block_table, const int32_t* positions, int num_seqs, int q_len,
                       int num_kv_heads, int head_dim, int page_size, int max_blocks_per_seq,
                       int num_pages, void* stream) {
  if (q_len < 1) return fail(GQA_ERR_INVALID_ARG, "q_len %d < 1", q_len);
  if (num_seqs < 0) return fail(GQA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_kv_heads < 1 || head_dim < 1 || page_size < 1 || max_blocks_per_seq < 1 || num_pages < 1)
    return fail(GQA_ERR_INVALID_ARG, "sizes must be positive");
  if (head_dim % 8 != 0) return fail(GQA_ERR_UNSUPPORTED, "head_dim must be a multiple of 8");
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size > INT32_MAX)
    return fail(GQA_ERR_UNSUPPORTED, "max_blocks_per_seq * page_size exceeds 2^31");
  if (num_seqs == 0) return GQA_OK;
  if (!k_new || !v_new || !k_pages || !v_pages || !block_table || !positions)
    return fail(GQA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16))
    return fail(GQA_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
  DeviceState* st;
  int dev;
  gqa_status s = get_state(&st, &dev);
  if (s != GQA_OK) return s;
  gqa::AppendParams p;
  p.k_new = static_cast<const uint4*>(k_new);
  p.v_new = static_cast<const uint4*>(v_new);
  p.k_pages = static_cast<uint4*>(k_pages);
  p.v_pages = static_cast<uint4*>(v_pages);
  p.block_table = block_table;
  p.positions = positions;
  p.err = st->err;
  p.num_seqs = num_seqs;
  p.num_kv_heads = num_kv_heads;
  p.vec_per_row = head_dim / 8;
  p.page_size = page_size;
  p.max_blocks = max_blocks_per_seq;
  p.num_pages = num_pages;
  p.q_len = q_len;
  cudaError_t e = gqa::launch_kv_append(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kv_append launch");
  g_launches.fetch_add(1);
  return GQA_OK;
}

gqa_status append_fp8_impl(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                           const float* k_scales, const float* v_scales, const int32_t* block_table,
                           const int32_t* positions, int num_seqs, int num_kv_heads, int head_dim, int page_size,
                           int max_blocks_per_seq, int num_pages, void* stream) {
  if (num_seqs < 0) return fail(GQA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_kv_heads < 1 || head_dim < 1 || page_size < 1 || max_blocks_per_seq < 1 || num_pages < 1)
    return fail(GQA_ERR_INVALID_ARG, "sizes must be positive");
  if (head_dim % 16 != 0) return fail(GQA_ERR_UNSUPPORTED, "head_dim must be a multiple of 16");
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size > INT32_MAX)
    return fail(GQA_ERR_UNSUPPORTED, "max_blocks_per_seq * page_size exceeds 2^31");
  if (num_seqs == 0) return GQA_OK;
  if (!k_new || !v_new || !k_pages || !v_pages || !k_scales || !v_scales || !block_table || !positions)
    return fail(GQA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16))
    return fail(GQA_ERR_INVALID_ARG, "k_new, v_new and the pools must be 16-byte aligned");
  if (!aligned(k_scales, 4) || !aligned(v_scales, 4))
    return fail(GQA_ERR_INVALID_ARG, "k_scales / v_scales must be 4-byte aligned");
  DeviceState* st;
  int dev;
  gqa_status s = get_state(&st, &dev);
  if (s != GQA_OK) return s;
  gqa::AppendFp8Params p{};
  p.k_new = static_cast<const uint4*>(k_new);
  p.v_new = static_cast<const uint4*>(v_new);
  p.k_pages = static_cast<uint4*>(k_pages);
  p.v_pages = static_cast<uint4*>(v_pages);
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.block_table = block_table;
  p.positions = positions;
  p.err = st->err;
  p.num_seqs = num_seqs;
  p.num_kv_heads = num_kv_heads;
  p.groups_per_row = head_dim / 16;
  p.page_size = page_size;
  p.max_blocks = max_blocks_per_seq;
  p.num_pages = num_pages;
  cudaError_t e = gqa::launch_kv_append_fp8(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kv_append_fp8 launch");
  g_launches.fetch_add(1);
  return GQA_OK;
}

}  // namespace

extern "C" {

const char* gqa_last_error_string(void) { return g_err_msg; }

int gqa_abi_version(void) { return 1; }

uint64_t gqa_launch_count(void) { return g_launches.load(); }

size_t gqa_kv_cache_bytes(int num_layers, int num_kv_heads, int head_dim, int64_t seq_len) {
  if (num_layers < 0 || num_kv_heads < 0 || head_dim < 0 || seq_len < 0) return 0;
  return static_cast<size_t>(2) * num_layers * num_kv_heads * head_dim *
         static_cast<size_t>(seq_len) * 2;
}

gqa_status gqa_set_num_workers(int n) {
  if (n < 0 || n > (1 << 20)) return fail(GQA_ERR_INVALID_ARG, "num_workers must be in [0, 2^20]");
  g_num_workers.store(n);
  return GQA_OK;
}

gqa_status gqa_set_wait_limit_ns(int64_t limit_ns, int arm_without_copy) {
  if (limit_ns <= 0) return fail(GQA_ERR_INVALID_ARG, "wait limit must be positive");
  g_wait_limit_ns.store(limit_ns);
  g_arm_without_copy.store(arm_without_copy ? 1 : 0);
  return GQA_OK;
}

gqa_status gqa_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                         const int32_t* block_table, const int32_t* positions, int num_seqs,
                         int num_kv_heads, int head_dim, int page_size, int max_blocks_per_seq,
                         int num_pages, void* stream) {
  return append_impl(k_new, v_new, k_pages, v_pages, block_table, positions, num_seqs, 1, num_kv_heads,
                     head_dim, page_size, max_blocks_per_seq, num_pages, stream);
}

gqa_status gqa_kv_append_multi(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                               const int32_t* block_table, const int32_t* positions, int num_seqs,
                               int q_len, int num_kv_heads, int head_dim, int page_size,
                               int max_blocks_per_seq, int num_pages, void* stream) {
  return append_impl(k_new, v_new, k_pages, v_pages, block_table, positions, num_seqs, q_len,
                     num_kv_heads, head_dim, page_size, max_blocks_per_seq, num_pages, stream);
}

gqa_status gqa_paged_decode_attn(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seq_lens, void* out,
                                 int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int page_size, float scale, int max_blocks_per_seq,
                                 int num_pages, void* stream) {
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads,
                     num_kv_heads, head_dim, page_size, scale, max_blocks_per_seq, num_pages,
                     stream, false);
}

gqa_status gqa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_pages,
                           void* v_pages, const int32_t* block_table, const int32_t* positions,
                           const int32_t* seq_lens, void* out, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int page_size, float scale,
                           int max_blocks_per_seq, int num_pages, void* stream) {
  gqa_status s = gqa_kv_append(k_new, v_new, k_pages, v_pages, block_table, positions, num_seqs,
                               num_kv_heads, head_dim, page_size, max_blocks_per_seq, num_pages,
                               stream);
  if (s != GQA_OK) return s;
  // The decode launch overlaps the append kernel's tail: the append writes only the
  // new K/V rows, which the decode's producer reads after waiting for it.
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads,
                     num_kv_heads, head_dim, page_size, scale, max_blocks_per_seq, num_pages,
                     stream, true);
}

gqa_status gqa_paged_multi_query_attn(const void* q, const void* k_pages, const void* v_pages,
                                      const int32_t* block_table, const int32_t* seq_lens, void* out,
                                      int num_seqs, int q_len, int num_heads, int num_kv_heads,
                                      int head_dim, int page_size, float scale, int max_blocks_per_seq,
                                      int num_pages, void* stream) {
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads,
                     num_kv_heads, head_dim, page_size, scale, max_blocks_per_seq, num_pages,
                     stream, false, q_len);
}

gqa_status gqa_multi_query_step(const void* q, const void* k_new, const void* v_new, void* k_pages,
                                void* v_pages, const int32_t* block_table, const int32_t* positions,
                                const int32_t* seq_lens, void* out, int num_seqs, int q_len,
                                int num_heads, int num_kv_heads, int head_dim, int page_size,
                                float scale, int max_blocks_per_seq, int num_pages, void* stream) {
  if (q_len < 1) return fail(GQA_ERR_INVALID_ARG, "q_len %d < 1", q_len);
  if (num_kv_heads >= 1 && num_heads % num_kv_heads == 0 &&
      static_cast<int64_t>(num_heads / num_kv_heads) * q_len > 128 && q_len > 1)
    return fail(GQA_ERR_UNSUPPORTED, "q_len %d x %d query heads per kv head exceeds 128", q_len,
                num_heads / num_kv_heads);
  gqa_status s = append_impl(k_new, v_new, k_pages, v_pages, block_table, positions, num_seqs, q_len,
                             num_kv_heads, head_dim, page_size, max_blocks_per_seq, num_pages, stream);
  if (s != GQA_OK) return s;
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads,
                     num_kv_heads, head_dim, page_size, scale, max_blocks_per_seq, num_pages,
                     stream, true, q_len);
}

gqa_status gqa_kv_quantize_fp8(const void* src, void* dst, const float* scales, int num_pages,
                               int num_kv_heads, int page_size, int head_dim, void* stream) {
  if (num_pages < 0) return fail(GQA_ERR_INVALID_ARG, "num_pages < 0");
  if (num_kv_heads < 1 || page_size < 1 || head_dim < 1) return fail(GQA_ERR_INVALID_ARG, "sizes must be positive");
  if (head_dim % 16 != 0) return fail(GQA_ERR_UNSUPPORTED, "head_dim must be a multiple of 16");
  if (num_pages == 0) return GQA_OK;
  if (!src || !dst || !scales) return fail(GQA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(scales, 4))
    return fail(GQA_ERR_INVALID_ARG, "src and dst must be 16-byte and scales 4-byte aligned");
  const int64_t groups = static_cast<int64_t>(num_pages) * num_kv_heads * page_size * (head_dim / 16);
  cudaError_t e = gqa::launch_kv_quantize(static_cast<const uint4*>(src), static_cast<uint4*>(dst), scales, groups,
                                          head_dim / 16, page_size, num_kv_heads, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kv_quantize launch");
  g_launches.fetch_add(1);
  return GQA_OK;
}

gqa_status gqa_kv_append_fp8(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const float* k_scales, const float* v_scales, const int32_t* block_table,
                             const int32_t* positions, int num_seqs, int num_kv_heads, int head_dim, int page_size,
                             int max_blocks_per_seq, int num_pages, void* stream) {
  return append_fp8_impl(k_new, v_new, k_pages, v_pages, k_scales, v_scales, block_table, positions, num_seqs,
                         num_kv_heads, head_dim, page_size, max_blocks_per_seq, num_pages, stream);
}

gqa_status gqa_paged_decode_attn_fp8(const void* q, const void* k_pages, const void* v_pages, const float* k_scales,
                                     const float* v_scales, const int32_t* block_table, const int32_t* seq_lens,
                                     void* out, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int page_size, float scale, int max_blocks_per_seq, int num_pages,
                                     void* stream) {
  if (!k_scales || !v_scales) return fail(GQA_ERR_INVALID_ARG, "k_scales and v_scales are required");
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads, num_kv_heads, head_dim,
                     page_size, scale, max_blocks_per_seq, num_pages, stream, false, 1, k_scales, v_scales);
}

gqa_status gqa_decode_step_fp8(const void* q, const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                               const float* k_scales, const float* v_scales, const int32_t* block_table,
                               const int32_t* positions, const int32_t* seq_lens, void* out, int num_seqs,
                               int num_heads, int num_kv_heads, int head_dim, int page_size, float scale,
                               int max_blocks_per_seq, int num_pages, void* stream) {
  if (!k_scales || !v_scales) return fail(GQA_ERR_INVALID_ARG, "k_scales and v_scales are required");
  gqa_status s = append_fp8_impl(k_new, v_new, k_pages, v_pages, k_scales, v_scales, block_table, positions,
                                 num_seqs, num_kv_heads, head_dim, page_size, max_blocks_per_seq, num_pages, stream);
  if (s != GQA_OK) return s;
  return decode_impl(q, k_pages, v_pages, block_table, seq_lens, out, num_seqs, num_heads, num_kv_heads, head_dim,
                     page_size, scale, max_blocks_per_seq, num_pages, stream, true, 1, k_scales, v_scales);
}

gqa_status gqa_paged_decode_attn_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         void* out, int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int page_size, float scale,
                                         int max_blocks_per_seq, int num_pages, void* stream) {
  if (num_seqs < 0) return fail(GQA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_heads < 1 || num_kv_heads < 1 || head_dim < 1 || page_size < 1 ||
      max_blocks_per_seq < 1 || num_pages < 1)
    return fail(GQA_ERR_INVALID_ARG, "sizes must be positive");
  if (num_heads % num_kv_heads != 0)
    return fail(GQA_ERR_INVALID_ARG, "num_heads (%d) is not a multiple of num_kv_heads (%d)",
                num_heads, num_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(GQA_ERR_UNSUPPORTED, "head_dim %d not built (64, 128)", head_dim);
  if (page_size % gqa::kChunk != 0 || page_size > 256)
    return fail(GQA_ERR_UNSUPPORTED, "page_size %d not built (multiple of 16, <= 256)", page_size);
  if (!std::isfinite(scale)) return fail(GQA_ERR_INVALID_ARG, "scale is not finite");
  const int64_t rows = static_cast<int64_t>(num_pages) * num_kv_heads * page_size;
  if (rows >= (int64_t{1} << 31))
    return fail(GQA_ERR_UNSUPPORTED, "num_pages * num_kv_heads * page_size exceeds 2^31");
  if (static_cast<int64_t>(max_blocks_per_seq) * page_size >= (int64_t{1} << 31))
    return fail(GQA_ERR_UNSUPPORTED, "max_blocks_per_seq * page_size exceeds 2^31");
  if (num_seqs == 0) return GQA_OK;
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out)
    return fail(GQA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(k_pages, 16) || !aligned(v_pages, 16))
    return fail(GQA_ERR_INVALID_ARG, "k_pages / v_pages must be 16-byte aligned");
  if (!aligned(q, 16) || !aligned(out, 8))
    return fail(GQA_ERR_INVALID_ARG, "q must be 16-byte and out 8-byte aligned");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  unsigned char* scratch = nullptr;
  int sms = 0;
  gqa_status s = noalloc_scratch(dev, &scratch, &sms);
  if (s != GQA_OK) return s;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);

  const int group = num_heads / num_kv_heads;
  const gqa::DecodePlan plan = gqa::plan_decode(head_dim, group);
  const size_t segments = static_cast<size_t>(num_seqs) * num_kv_heads * plan.n_ht;
  if (segments > kNoAllocMaxSegments)
    return fail(GQA_ERR_UNSUPPORTED,
                "allocation-free decode holds at most %zu segments (num_seqs * num_kv_heads * "
                "head tiles); this call needs %zu",
                kNoAllocMaxSegments, segments);
  const int64_t blocks_per_seq =
      (static_cast<int64_t>(max_blocks_per_seq) * page_size + gqa::kBlock - 1) / gqa::kBlock;
  const int64_t max_blocks = static_cast<int64_t>(num_seqs) * num_kv_heads * plan.n_ht * blocks_per_seq;
  int64_t workers = static_cast<int64_t>(sms) * plan.ctas_per_sm;
  const int forced = g_num_workers.load();
  if (forced > 0) workers = forced;
  if (workers > max_blocks) workers = max_blocks;
  if (workers < 1) workers = 1;
  // Fewer workers when the split partials of every worker would not fit the array.
  const size_t fixed = kNoAllocHeaderBytes + align256(segments * sizeof(int32_t));
  const size_t per_worker = 2 * static_cast<size_t>(plan.heads_per_seg) *
                            (static_cast<size_t>(head_dim) + 2) * sizeof(float) + 512;
  const int64_t fit = static_cast<int64_t>((kNoAllocScratchBytes - fixed) / per_worker);
  if (fit < 1)
    return fail(GQA_ERR_UNSUPPORTED, "allocation-free scratch (%zu bytes) is too small for this call",
                kNoAllocScratchBytes);
  if (workers > fit) workers = fit;
  const size_t slots = static_cast<size_t>(2 * workers);
  unsigned char* counters = scratch + kNoAllocHeaderBytes;
  unsigned char* part_ml = scratch + fixed;
  unsigned char* part_o = part_ml + align256(slots * plan.heads_per_seg * 2 * sizeof(float));
  if (part_o + slots * plan.heads_per_seg * head_dim * sizeof(float) > scratch + kNoAllocScratchBytes)
    return fail(GQA_ERR_UNSUPPORTED, "allocation-free scratch layout does not fit");
  // The array keeps the previous call's contents: the arrival counters must start at
  // zero (a call that timed out may leave them set).  The error word is not cleared
  // here: it accumulates until gqa_check_device_error reads and clears it.
  e = cudaMemsetAsync(counters, 0, segments * sizeof(int32_t), strm);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(allocation-free scratch)");


  gqa::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.part_o = reinterpret_cast<float*>(part_o);
  p.part_ml = reinterpret_cast<float*>(part_ml);
  p.counters = reinterpret_cast<int32_t*>(counters);
  p.err = reinterpret_cast<uint32_t*>(scratch);
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.n_ht = plan.n_ht;
  p.heads_per_seg = plan.heads_per_seg;
  p.page_size = page_size;
  p.max_blocks = max_blocks_per_seq;
  p.num_pages = num_pages;
  p.head_dim = head_dim;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_workers = static_cast<int>(workers);
  p.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns.load());
  p.arm_without_copy = g_arm_without_copy.load();
  p.q_len = 1;
  e = launch_with_maps(p, plan, q, k_pages, v_pages, rows, dev, static_cast<int>(workers), strm,
                       false, &s);
  if (s != GQA_OK) return s;
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  g_launches.fetch_add(plan.tensor_cores && workers > 1 ? 2 : 1);
  return GQA_OK;
}

gqa_status gqa_check_device_error(void* stream) {
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(strm);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  // Two error words may exist on this device: the workspace's (every call but the
  // allocation-free decode) and the one in the allocation-free call's fixed array.
  // Only words that calls have set up are read; nothing is allocated here.
  uint32_t word = 0;
  DeviceState* st = existing_state(dev);
  if (st != nullptr) {
    uint32_t w = 0;
    e = cudaMemcpy(&w, st->err, sizeof(w), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
    if (w != 0) {
      e = cudaMemset(st->err, 0, sizeof(uint32_t));
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error word)");
    }
    word |= w;
  }
  unsigned char* na = noalloc_scratch_if_set_up(dev);
  if (na != nullptr) {
    uint32_t w = 0;
    e = cudaMemcpy(&w, na, sizeof(w), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(allocation-free error word)");
    if (w != 0) {
      e = cudaMemset(na, 0, sizeof(uint32_t));
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(allocation-free error word)");
    }
    word |= w;
  }
  if (word == 0) return GQA_OK;
  if (word & gqa::kErrTimeout) {
    // A timed-out launch may leave workspace arrival counters set (the allocation-free
    // call clears its own at every call).
    if (st != nullptr) {
      std::lock_guard<std::mutex> lk(g_mu);
      if (st->counters) cudaMemset(st->counters, 0, st->counters_cap * sizeof(int32_t));
    }
    cudaDeviceSynchronize();
    return fail(GQA_ERR_TIMEOUT, "a kernel wait ran out of time; its work was skipped");
  }
  return fail(GQA_ERR_DEVICE_BOUNDS,
              "a page id, position or sequence length was out of range; that work was skipped");
}

}  // extern "C"
