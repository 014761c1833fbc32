// Shared declarations between the C-ABI host code and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gqa_decode.h"

namespace gqa {

// Sets the calling thread's gqa_last_error_string() text and returns s.
gqa_status set_error(gqa_status s, const char* fmt, ...);

// Bits of the per-device error word.
enum : uint32_t {
  kErrBounds = 1u,   // page id / position / length out of range: work skipped
  kErrTimeout = 2u,  // a bounded wait ran out: work skipped
};

// Tokens per TMA sub-chunk: every supported page size is a multiple of it, so a
// sub-chunk never straddles two pages and is one contiguous [16, head_dim] tile of
// one (page, kv head).
constexpr int kChunk = 16;
// Tokens per pipeline stage (four sub-chunks): the unit the work list is cut into.
constexpr int kBlock = 64;
constexpr int kSubChunks = kBlock / kChunk;
// Most query heads one segment (kv head x head tile) covers; partial slots hold this many.
constexpr int kMaxSegHeads = 128;

// Rows of one K/V copy of the tcgen05 kernel: the largest power of two dividing the page
// size, at most one block, so a copy never straddles two pages and a block is a whole
// number of copies.
__host__ __device__ __forceinline__ int tc_box_rows(int page_size) {
  const int low = page_size & -page_size;
  return low < kBlock ? low : kBlock;
}

struct DecodeParams {
  const uint16_t* q;          // [B, H, D] bf16
  uint16_t* out;              // [B, H, D] bf16
  const int32_t* block_table; // [B, MB]
  const int32_t* seq_lens;    // [B]
  float* part_o;              // [2 * num_workers, heads_per_seg, D] fp32 (unnormalised)
  float* part_ml;             // [2 * num_workers, heads_per_seg, 2] fp32 (ref max, sum), log2
  int32_t* counters;          // [B * Hk * n_ht], zero between launches
  uint32_t* err;              // device error word
  int num_seqs, num_heads, num_kv_heads, group, n_ht, page_size, max_blocks, num_pages;
  int head_dim;
  int heads_per_seg;          // query heads one segment covers
  float scale_log2;           // scale * log2(e)
  int num_workers;            // CTAs the work list is split over
  uint64_t wait_limit_ns;
  int arm_without_copy;
  int q_len;                  // query tokens per sequence (q, out: [B, q_len, H, D]); 1 = decode
  // 8-bit cache: k_pages / v_pages hold e4m3 codes; a cached value is code * scale of its
  // kv head (k_scales, v_scales [Hk] fp32).  nullptr for a bf16 cache.
  const float* k_scales;
  const float* v_scales;
  // mma.sync kernel, e4m3 codes: 0 = separate K and V tensor maps; otherwise the K map
  // spans both pools with an outer coordinate of extent 2, one copy bringing a
  // sub-chunk's K and V: 1 = K at coordinate 0, V at 1; 2 = V at 0, K at 1 (the V pool
  // lies lower in memory).  Always 0 for a bf16 cache.
  int kv_pair;
  // floor(x / page_size) == umulhi(x, ps_magic) >> ps_shift for 0 <= x < 2^31.
  uint32_t ps_magic;
  int ps_shift;
};

// Multiply-and-shift constants of division by d (1 < d < 2^31) for dividends below
// 2^31, after Granlund and Montgomery, "Division by invariant integers using
// multiplication" (1994): with l = ceil(log2 d), m = ceil(2^(31 + l) / d) fits in 32 bits
// and m * d - 2^(31 + l) < d <= 2^l, so floor(x * m / 2^(31 + l)) == floor(x / d).
inline void divisor_magic(uint32_t d, uint32_t* magic, int* shift) {
  int l = 0;
  while ((uint64_t{1} << l) < d) ++l;
  const uint64_t num = uint64_t{1} << (31 + l);
  *magic = static_cast<uint32_t>((num + d - 1) / d);
  *shift = l - 1;  // umulhi already drops 32 of the 31 + l bits
}

#ifdef __CUDACC__
__device__ __forceinline__ int fast_div(int x, uint32_t magic, int shift) {
  return static_cast<int>(__umulhi(static_cast<uint32_t>(x), magic) >> shift);
}
#endif

struct AppendParams {
  const uint4* k_new;
  const uint4* v_new;
  uint4* k_pages;
  uint4* v_pages;
  const int32_t* block_table;
  const int32_t* positions;
  uint32_t* err;
  int num_seqs, num_kv_heads, vec_per_row, page_size, max_blocks, num_pages;
  int q_len;                  // rows per sequence: k_new [B, q_len, Hk, D] to positions[b] + i
};

// The append into an 8-bit (e4m3) cache: 16 elements per thread.
struct AppendFp8Params {
  const uint4* k_new;         // [B, Hk, D] bf16
  const uint4* v_new;
  uint4* k_pages;             // [P, Hk, ps, D] e4m3
  uint4* v_pages;
  const float* k_scales;      // [Hk]
  const float* v_scales;
  const int32_t* block_table;
  const int32_t* positions;
  uint32_t* err;
  int num_seqs, num_kv_heads, groups_per_row, page_size, max_blocks, num_pages;
};

// Launchers (return the cudaError_t of the launch).
cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream);
cudaError_t launch_kv_append_fp8(const AppendFp8Params& p, cudaStream_t stream);
// Codes of a bf16 pool, groups of 16 elements (groups_per_row = head_dim / 16).
cudaError_t launch_kv_quantize(const uint4* src, uint4* dst, const float* scales, int64_t groups,
                               int groups_per_row, int page_size, int num_kv_heads, cudaStream_t stream);

// How a (head_dim, group) problem is mapped onto the decode kernel.
struct DecodePlan {
  int tensor_cores;   // 1: tcgen05 kernel (large groups), 0: mma.sync warp-specialized kernel
  int n_tiles;        // 8-head MMA n-tiles per consumer
  int consumers;      // consumer (MMA) warps per CTA; one producer warp is added
  int heads_per_seg;  // query heads a segment covers
  int n_ht;           // segments per kv head
  int stages;         // pipeline stages per CTA
  int ctas_per_sm;
  size_t smem_bytes;
};

// group: query rows per kv head; mq_rows: they are several query tokens' heads; fp8: the
// cache holds e4m3 codes.
DecodePlan plan_decode(int head_dim, int group, bool mq_rows = false, bool fp8 = false);
// overlap_previous: launch with programmatic stream serialization, so the prologue
// overlaps the preceding kernel of the stream (which must write nothing the decode reads
// except the K/V pools); the producer waits for that kernel before its first K/V copy.
// tcgen05 kernel: K/V maps with boxes of tc_box_rows(page_size) rows x 64 columns and
// every column group when that is 64 rows, one group otherwise; Q map over
// [num_seqs * num_heads, head_dim] with boxes of 128 rows x every column group.
cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tq, int grid, cudaStream_t stream, bool overlap);
size_t decode_tc_smem_bytes(int head_dim, bool fp8 = false);

cudaError_t launch_decode(const DecodeParams& p, const DecodePlan& plan, const CUtensorMap& tmap_k,
                          const CUtensorMap& tmap_v, int grid, cudaStream_t stream,
                          bool overlap_previous = false);

}  // namespace gqa
