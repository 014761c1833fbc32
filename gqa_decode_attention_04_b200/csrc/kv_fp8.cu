// Writing into an 8-bit (e4m3) K/V cache: quantise a whole bf16 pool, and the decode
// step's append of one new row per (sequence, kv head).
//
// The TensorRT MQA page calibrates Q, K and V separately with their own per-tensor
// scales in 8-bit mode; here K and V each carry one fp32 scale per kv head (a per-tensor
// scale is the case of equal scales).  A stored code is the e4m3 value nearest to the
// fp32 quotient x / scale (IEEE division, round to nearest even), saturating to +-448;
// NaN stays NaN.  One thread handles 16 consecutive elements of one row: 32 bytes of
// bf16 in, 16 bytes of codes out.
#include <cuda_fp8.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

namespace {

// Two bf16 (one 32-bit word, element 0 in the low half) divided by s -> two codes
// (element 0 in the low byte).
__device__ __forceinline__ uint32_t quantize2(uint32_t w, float s) {
  float2 f;
  f.x = __fdiv_rn(__uint_as_float(w << 16), s);
  f.y = __fdiv_rn(__uint_as_float(w & 0xffff0000u), s);
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3));
}

// 16 bf16 values (a: elements 0-7, b: 8-15) -> 16 codes.
__device__ __forceinline__ uint4 quantize16(const uint4 a, const uint4 b, float s) {
  uint4 o;
  o.x = quantize2(a.x, s) | (quantize2(a.y, s) << 16);
  o.y = quantize2(a.z, s) | (quantize2(a.w, s) << 16);
  o.z = quantize2(b.x, s) | (quantize2(b.y, s) << 16);
  o.w = quantize2(b.z, s) | (quantize2(b.w, s) << 16);
  return o;
}

}  // namespace

__global__ void __launch_bounds__(256) kv_quantize_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          const float* __restrict__ scales, int64_t groups,
                                                          int groups_per_row, int page_size, int num_kv_heads) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= groups) return;
  const int64_t row = g / groups_per_row;  // (page * Hk + kvh) * page_size + slot
  const int kvh = static_cast<int>((row / page_size) % num_kv_heads);
  const float s = __ldg(scales + kvh);
  dst[g] = quantize16(__ldg(src + 2 * g), __ldg(src + 2 * g + 1), s);
}

__global__ void __launch_bounds__(256) kv_append_fp8_kernel(const AppendFp8Params p) {
  // A decode launched right after this one may start its prologue now; it reads none of
  // what this kernel writes before waiting for this grid to complete.
  ptx::pdl_launch_dependents();
  const int64_t per_tensor = static_cast<int64_t>(p.num_seqs) * p.num_kv_heads * p.groups_per_row;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= 2 * per_tensor) return;
  const bool is_v = idx >= per_tensor;
  const int64_t r = is_v ? idx - per_tensor : idx;
  const int grp = static_cast<int>(r % p.groups_per_row);
  const int64_t row = r / p.groups_per_row;  // b * Hk + kvh
  const int kvh = static_cast<int>(row % p.num_kv_heads);
  const int b = static_cast<int>(row / p.num_kv_heads);

  const int pos = __ldg(p.positions + b);
  if (pos < 0 || static_cast<int64_t>(pos) >= static_cast<int64_t>(p.max_blocks) * p.page_size) {
    if (grp == 0 && kvh == 0 && !is_v) atomicOr(p.err, kErrBounds);
    return;
  }
  const int page = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + pos / p.page_size);
  if (page < 0 || page >= p.num_pages) {
    if (grp == 0 && kvh == 0 && !is_v) atomicOr(p.err, kErrBounds);
    return;
  }
  const int64_t dst =
      ((static_cast<int64_t>(page) * p.num_kv_heads + kvh) * p.page_size + pos % p.page_size) * p.groups_per_row + grp;
  const uint4* src = (is_v ? p.v_new : p.k_new) + 2 * r;
  const float s = __ldg((is_v ? p.v_scales : p.k_scales) + kvh);
  (is_v ? p.v_pages : p.k_pages)[dst] = quantize16(__ldg(src), __ldg(src + 1), s);
}

cudaError_t launch_kv_quantize(const uint4* src, uint4* dst, const float* scales, int64_t groups,
                               int groups_per_row, int page_size, int num_kv_heads, cudaStream_t stream) {
  if (groups == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (groups + threads - 1) / threads;
  kv_quantize_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(src, dst, scales, groups,
                                                                            groups_per_row, page_size, num_kv_heads);
  return cudaGetLastError();
}

cudaError_t launch_kv_append_fp8(const AppendFp8Params& p, cudaStream_t stream) {
  const int64_t n = 2LL * p.num_seqs * p.num_kv_heads * p.groups_per_row;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  kv_append_fp8_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace gqa
