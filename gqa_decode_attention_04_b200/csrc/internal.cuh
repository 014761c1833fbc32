// Shared declarations between the C-ABI host code and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gqa {

// Bits of the per-device error word.
enum : uint32_t {
  kErrBounds = 1u,   // page id / position / length out of range: work skipped
  kErrTimeout = 2u,  // a bounded wait ran out: work skipped
};

// Tokens per pipeline chunk: every supported page size is a multiple of it, so a
// chunk never straddles two pages and is one contiguous [16, head_dim] tile of
// one (page, kv head).
constexpr int kChunk = 16;

// Query heads handled per head tile (the M dimension of one m16n8k16 MMA).
constexpr int kHeadTile = 16;

struct DecodeParams {
  const uint16_t* q;          // [B, H, D] bf16
  uint16_t* out;              // [B, H, D] bf16
  const int32_t* block_table; // [B, MB]
  const int32_t* seq_lens;    // [B]
  float* part_o;              // [2 * num_workers, kHeadTile, D] fp32 (unnormalised)
  float* part_ml;             // [2 * num_workers, kHeadTile, 2] fp32 (max, sum), log2 domain
  int32_t* counters;          // [B * Hk * n_ht], zero between launches
  uint32_t* err;              // device error word
  int num_seqs, num_heads, num_kv_heads, group, n_ht, page_size, max_blocks, num_pages;
  int head_dim;
  float scale_log2;           // scale * log2(e)
  int num_workers;
  uint64_t wait_limit_ns;
  int arm_without_copy;
};

struct AppendParams {
  const uint4* k_new;
  const uint4* v_new;
  uint4* k_pages;
  uint4* v_pages;
  const int32_t* block_table;
  const int32_t* positions;
  uint32_t* err;
  int num_seqs, num_kv_heads, vec_per_row, page_size, max_blocks, num_pages;
};

// Launchers (return the cudaError_t of the launch).
cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t stream);

struct DecodeLaunch {
  int warps_per_cta;
  int ctas_per_sm;
  size_t smem_bytes;
};

// Kernel configuration for a head_dim / group combination.
DecodeLaunch decode_launch_config(int head_dim, int group);
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmap_k,
                          const CUtensorMap& tmap_v, int grid, cudaStream_t stream);

}  // namespace gqa
