// kv_append: scatter each sequence's new K/V row (or q_len rows, to consecutive
// positions) into its page slot.
//
// The "scatter" half of paged KV strategy 1 on the tiny-llm "优化" page (block
// table + scatter/gather); the decode step's append position.  One thread moves
// one 16-byte vector, so a warp writes 512 contiguous bytes of one slot row
// (head_dim = 128: two rows per warp) and the copy is bit-exact.
#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
  // A decode kernel launched right after this one may start its prologue (it reads
  // none of what this kernel writes until it waits for this grid to complete).
  ptx::pdl_launch_dependents();
  const int64_t per_tensor =
      static_cast<int64_t>(p.num_seqs) * p.q_len * p.num_kv_heads * p.vec_per_row;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= 2 * per_tensor) return;
  const bool is_v = idx >= per_tensor;
  const int64_t r = is_v ? idx - per_tensor : idx;
  const int vec = static_cast<int>(r % p.vec_per_row);
  const int64_t row = r / p.vec_per_row;  // (b * q_len + i) * Hk + kvh
  const int kvh = static_cast<int>(row % p.num_kv_heads);
  const int64_t bi = row / p.num_kv_heads;
  const int b = static_cast<int>(bi / p.q_len);
  const int i = static_cast<int>(bi - static_cast<int64_t>(b) * p.q_len);

  const int pos0 = __ldg(p.positions + b);
  const int64_t pos = static_cast<int64_t>(pos0) + i;
  if (pos0 < 0 || pos >= static_cast<int64_t>(p.max_blocks) * p.page_size) {
    if (vec == 0 && kvh == 0 && !is_v) atomicOr(p.err, kErrBounds);
    return;
  }
  const int page = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + pos / p.page_size);
  if (page < 0 || page >= p.num_pages) {
    if (vec == 0 && kvh == 0 && !is_v) atomicOr(p.err, kErrBounds);
    return;
  }
  const int64_t dst =
      ((static_cast<int64_t>(page) * p.num_kv_heads + kvh) * p.page_size + pos % p.page_size) *
          p.vec_per_row + vec;
  const uint4 v = is_v ? __ldg(p.v_new + r) : __ldg(p.k_new + r);
  (is_v ? p.v_pages : p.k_pages)[dst] = v;
}

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream) {
  const int64_t n = 2LL * p.num_seqs * p.q_len * p.num_kv_heads * p.vec_per_row;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  kv_append_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace gqa
