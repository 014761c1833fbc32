// Paged GQA/MQA decode attention: one new query token per sequence.
//
// What is computed (page "TensorRT对Multi-Query Attention的专项优化支持": decode re-reads
// all cached K/V; MQA/GQA query heads share K/V heads; QK^T then AV on tensor cores with
// tiled shared-memory K/V prefetch; paged cache.  tiny-llm "优化" page: GQA, block table
// + gather, FlashDecoding for long contexts):
//
//   out[b, h] = sum_t softmax_t(scale * q[b, h] . K_b[t, kvh]) V_b[t, kvh],  kvh = h / G.
//
// Design (B200, sm_100a):
//   * Work space.  The context of every (sequence b, segment s = kv head x head tile)
//     is cut into 16-token chunks; all chunks of all segments form one linear list in
//     (b, s, chunk) order.  The list is split into num_workers equal ranges, one per
//     warp, so every warp streams the same number of K/V bytes whatever the length mix
//     (the split-KV / FlashDecoding idea, balanced at chunk granularity).  Every CTA
//     derives the split itself from seq_lens: no planning kernel, no host sync.
//   * Loads.  One lane of each warp issues 2-D TMA copies of the chunk's K and V tiles
//     ([16 tokens, 64 dims] boxes, 128-byte swizzle) into a per-warp ring of stages,
//     completion counted on an mbarrier; page ids come from the block table one chunk
//     ahead.  Each chunk is one contiguous 16*D*2-byte run of HBM per tensor.
//   * Math.  A kv head's whole query group (up to 16 heads) is the M=16 side of
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate): S = Q K^T reads each K row once for
//     all G heads; P V likewise reads V once.  Online softmax keeps a running max and
//     sum per head row in registers (quad shuffles), in the log2 domain.
//   * Merge.  A segment whose chunks fall in one warp's range is written straight to
//     out.  Otherwise each warp stores its piece (unnormalised o, max, sum) and bumps
//     the segment's arrival counter; the last arriver merges all pieces with their
//     log-sum-exp weights, writes out and resets the counter to zero.
//   * Safety.  Page ids, lengths and positions are range-checked on the device (bad
//     work is skipped and an error bit set); every mbarrier wait is bounded in time.
#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

namespace {

template <int D>
struct Geo {
  static constexpr int kBoxes = D / 64;               // 64-column (128-byte) boxes per row
  static constexpr int kBoxBytes = kChunk * 128;      // 16 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile + V tile
};

// Byte offset of 16-byte column chunk `cc` (0 .. D/8-1) of row `r` (0..15) in a tile
// written by TMA with 128-byte swizzling: within each 1024-byte atom the chunk index
// is XORed with the row index modulo 8.
__device__ __forceinline__ uint32_t sw128(int r, int cc) {
  return static_cast<uint32_t>((cc >> 3) * 2048 + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ int eff_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

struct Cursor {
  int b;        // sequence
  int seg;      // kv_head * n_ht + head_tile
  int c;        // chunk within the segment
  int nchunks;  // chunks per segment of sequence b
  int len;      // effective context length of sequence b
};

__device__ __forceinline__ void cursor_load_seq(Cursor& cu, const DecodeParams& p, int cap) {
  cu.len = (cu.b >= 0 && cu.b < p.num_seqs) ? eff_len(__ldg(p.seq_lens + cu.b), cap) : 0;
  cu.nchunks = (cu.len + kChunk - 1) / kChunk;
}

// Step to the next chunk of the linear work list (only called while chunks remain).
__device__ __forceinline__ void cursor_next(Cursor& cu, const DecodeParams& p, int segs, int cap) {
  if (++cu.c < cu.nchunks) return;
  cu.c = 0;
  if (++cu.seg < segs) return;
  cu.seg = 0;
  do {
    ++cu.b;
    cursor_load_seq(cu, p, cap);
  } while (cu.nchunks == 0 && cu.b + 1 < p.num_seqs);
}

__device__ __forceinline__ int64_t worker_start(int64_t w, int64_t T, int64_t W) { return w * T / W; }
// The worker whose range holds linear chunk x.
__device__ __forceinline__ int64_t worker_of(int64_t x, int64_t T, int64_t W) {
  return ((x + 1) * W - 1) / T;
}

}  // namespace

template <int D, int WARPS, int STAGES, bool HI>
__global__ void __launch_bounds__(WARPS * 32, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using G_ = Geo<D>;
  constexpr int KS = D / 16;  // k-steps of QK^T, also d-tile pairs of PV
  constexpr int NT = D / 8;   // n-tiles of the output accumulator

  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_red[WARPS];
  __shared__ int64_t s_x0[WARPS];
  __shared__ int s_start_b[WARPS];
  __shared__ int64_t s_start_base[WARPS];
  __shared__ int64_t s_wtot[WARPS];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int B = p.num_seqs;
  const int segs = p.num_kv_heads * p.n_ht;
  const int cap = p.max_blocks * p.page_size;

  // ---------------------------------------------------------------- prologue
  // Pass 1: total chunk count T (and zero rows of empty sequences).
  int64_t mine = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = __ldg(p.seq_lens + b);
    const int Le = eff_len(L, cap);
    if ((L < 0 || L > cap) && blockIdx.x == 0) atomicOr(p.err, kErrBounds);
    if (Le == 0 && (b % gridDim.x) == blockIdx.x) {
      uint32_t* o = reinterpret_cast<uint32_t*>(p.out + static_cast<int64_t>(b) * p.num_heads * D);
      for (int i = 0; i < p.num_heads * D / 2; ++i) o[i] = 0u;
    }
    mine += static_cast<int64_t>((Le + kChunk - 1) / kChunk) * segs;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if (lane == 0) s_red[warp] = mine;
  __syncthreads();
  int64_t T = 0;
#pragma unroll
  for (int i = 0; i < WARPS; ++i) T += s_red[i];

  // With fewer chunks than workers only the first T workers get work, so every
  // worker in use owns at least one chunk and the pieces of a segment are exactly
  // the workers worker_of(first chunk) .. worker_of(last chunk).
  const int64_t W = min(static_cast<int64_t>(p.num_workers), T);
  if (W == 0) return;  // nothing to attend (all sequences empty)
  const int64_t w = static_cast<int64_t>(blockIdx.x) * WARPS + warp;
  const int64_t x0 = (w < W) ? worker_start(w, T, W) : T;
  const int64_t x1 = (w < W) ? worker_start(w + 1, T, W) : T;
  if (lane == 0) {
    s_x0[warp] = x0;
    s_start_b[warp] = -1;
  }
  __syncthreads();

  // Pass 2: locate the sequence holding each warp's first chunk (tiled block scan).
  {
    int64_t base = 0;
    int64_t need_max = -1;
#pragma unroll
    for (int i = 0; i < WARPS; ++i) need_max = max(need_max, s_x0[i] < T ? s_x0[i] : -1);
    for (int t0 = 0; t0 < B && base <= need_max; t0 += blockDim.x) {
      const int b = t0 + threadIdx.x;
      int64_t n = 0;
      if (b < B) n = static_cast<int64_t>((eff_len(__ldg(p.seq_lens + b), cap) + kChunk - 1) / kChunk) * segs;
      int64_t incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (lane == 31) s_wtot[warp] = incl;
      __syncthreads();
      int64_t pre = 0, tot = 0;
#pragma unroll
      for (int i = 0; i < WARPS; ++i) {
        if (i < warp) pre += s_wtot[i];
        tot += s_wtot[i];
      }
      incl += pre;
      const int64_t lo = base + incl - n, hi = base + incl;
      if (n > 0) {
#pragma unroll
        for (int i = 0; i < WARPS; ++i) {
          const int64_t xs = s_x0[i];
          if (xs >= lo && xs < hi) {
            s_start_b[i] = b;
            s_start_base[i] = lo;
          }
        }
      }
      base += tot;
      __syncthreads();
    }
  }
  __syncthreads();
  if (x0 >= x1) return;  // idle worker (fewer chunks than workers)

  // ---------------------------------------------------------------- per-warp state
  const uint32_t smem0 = ptx::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (smem0 & 1023u)) & 1023u;
  const uint32_t ring = smem0 + pad + static_cast<uint32_t>(warp * STAGES * G_::kStageBytes);
  const uint32_t bars = smem0 + pad + static_cast<uint32_t>(WARPS * STAGES * G_::kStageBytes) +
                        static_cast<uint32_t>(warp * STAGES * 8);

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) ptx::mbar_init(bars + 8 * s, 1);
    ptx::fence_mbarrier_init();
    ptx::prefetch_tensormap(&tmap_k);
    ptx::prefetch_tensormap(&tmap_v);
  }
  __syncwarp();
  const uint64_t policy = ptx::policy_evict_first();

  const int start_b = s_start_b[warp];
  const int64_t start_base = s_start_base[warp];
  if (start_b < 0) {  // cannot happen for a non-empty range; never index with it
    if (lane == 0) atomicOr(p.err, kErrBounds);
    return;
  }
  Cursor ci;  // issue cursor
  ci.b = start_b;
  cursor_load_seq(ci, p, cap);
  {
    const int64_t off = x0 - start_base;
    ci.seg = static_cast<int>(off / ci.nchunks);
    ci.c = static_cast<int>(off % ci.nchunks);
  }
  Cursor cc = ci;  // compute cursor
  const int64_t total = x1 - x0;

  auto page_of = [&](const Cursor& cu) -> int {
    if (cu.b >= p.num_seqs || cu.nchunks == 0) return -1;  // flagged as a bad page
    return __ldg(p.block_table + static_cast<int64_t>(cu.b) * p.max_blocks +
                 (cu.c * kChunk) / p.page_size);
  };

  uint32_t valid_bits = 0;  // bit s: stage s holds real data (page id was in range)
  int next_page = page_of(ci);
  int64_t issued = 0;

  auto issue = [&](int stage) {
    const int page = next_page;
    const bool ok = page >= 0 && page < p.num_pages;
    const uint32_t bar = bars + 8 * stage;
    if (ok) valid_bits |= 1u << stage; else valid_bits &= ~(1u << stage);
    if (lane == 0) {
      if (!ok) {
        atomicOr(p.err, kErrBounds);
        ptx::mbar_arrive(bar);
      } else {
        ptx::mbar_arrive_expect_tx(bar, G_::kStageBytes);
        if (!p.arm_without_copy) {
          const int kvh = ci.seg / p.n_ht;
          const int row = (page * p.num_kv_heads + kvh) * p.page_size + (ci.c * kChunk) % p.page_size;
          const uint32_t kdst = ring + stage * G_::kStageBytes;
          const uint32_t vdst = kdst + G_::kTileBytes;
#pragma unroll
          for (int bx = 0; bx < G_::kBoxes; ++bx) {
            ptx::tma_load_2d(kdst + bx * G_::kBoxBytes, &tmap_k, bar, bx * 64, row, policy);
            ptx::tma_load_2d(vdst + bx * G_::kBoxBytes, &tmap_v, bar, bx * 64, row, policy);
          }
        }
      }
    }
    ++issued;
    if (issued < total) {
      cursor_next(ci, p, segs, cap);
      next_page = page_of(ci);
    }
  };

  const int nfill = total < STAGES ? static_cast<int>(total) : STAGES;
  for (int s = 0; s < nfill; ++s) issue(s);

  // Fragment coordinates.
  const int q4 = lane & 3;   // column pair within an 8-wide n-tile
  const int r0 = lane >> 2;  // head row (r0 + 8 is the second row)

  uint32_t qf[KS][4];
  float o[NT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int nrows = 0;  // valid head rows of the current head tile

  auto load_q = [&](const Cursor& cu) {
    const int kvh = cu.seg / p.n_ht;
    const int ht = cu.seg % p.n_ht;
    nrows = min(kHeadTile, p.group - ht * kHeadTile);
    const int head0 = kvh * p.group + ht * kHeadTile;
    const uint32_t* qrow0 = reinterpret_cast<const uint32_t*>(
        p.q + (static_cast<int64_t>(cu.b) * p.num_heads + head0 + r0) * D);
    const uint32_t* qrow1 = reinterpret_cast<const uint32_t*>(
        p.q + (static_cast<int64_t>(cu.b) * p.num_heads + head0 + r0 + 8) * D);
    const bool v0 = r0 < nrows, v1 = HI && (r0 + 8 < nrows);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c0 = (ks * 16 + 2 * q4) / 2;
      qf[ks][0] = v0 ? __ldg(qrow0 + c0) : 0u;
      qf[ks][1] = v1 ? __ldg(qrow1 + c0) : 0u;
      qf[ks][2] = v0 ? __ldg(qrow0 + c0 + 4) : 0u;
      qf[ks][3] = v1 ? __ldg(qrow1 + c0 + 4) : 0u;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  };

  load_q(cc);
  int64_t piece_x = x0;          // linear index of the current piece's first chunk
  int piece_c0 = cc.c;           // its chunk index within the segment
  bool first_seg = true;
  const float sl2 = p.scale_log2;
  const uint64_t limit = p.wait_limit_ns;

  for (int64_t i = 0; i < total; ++i) {
    const int stage = static_cast<int>(i % STAGES);
    const uint32_t parity = static_cast<uint32_t>((i / STAGES) & 1);
    // Every lane observes the barrier itself (acquire); the outcome is made
    // warp-uniform so no lane computes while another gives up.
    const bool arrived = ptx::mbar_wait_bounded(bars + 8 * stage, parity, limit);
    if (!__all_sync(0xffffffffu, arrived)) {
      // Out of time: flag it, give in-flight copies a bounded chance to land, leave.
      if (lane == 0) atomicOr(p.err, kErrTimeout);
      for (int64_t j = i; j < issued; ++j) {
        const int st = static_cast<int>(j % STAGES);
        ptx::mbar_wait_bounded(bars + 8 * st, static_cast<uint32_t>((j / STAGES) & 1), limit);
      }
      return;
    }

    if (valid_bits & (1u << stage)) {
      const uint32_t kb = ring + stage * G_::kStageBytes;
      const uint32_t vb = kb + G_::kTileBytes;
      const int nvalid = cc.len - cc.c * kChunk;  // >= 1

      // S = Q K^T for 16 tokens: two 8-token n-tiles.
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int tok = ((lane >> 4) << 3) + (lane & 7);
        const int sub = (lane >> 3) & 1;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ptx::ldmatrix_x4(kb + sw128(tok, 2 * ks + sub), b0, b1, b2, b3);
          ptx::mma_bf16_16816(sc[0], qf[ks], b0, b1);
          ptx::mma_bf16_16816(sc[1], qf[ks], b2, b3);
        }
      }

      // Online softmax (log2 domain).
      if (nvalid < kChunk) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = nt * 8 + 2 * q4 + (e & 1);
            sc[nt][e] = (t < nvalid) ? sc[nt][e] * sl2 : -INFINITY;
          }
      } else {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] *= sl2;
      }
      uint32_t pa[4];
      {
        float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m0, mx);
        const float mu = (mn == -INFINITY) ? 0.f : mn;
        const float alpha = ptx::ex2(m0 - mu);
        const float p00 = ptx::ex2(sc[0][0] - mu), p01 = ptx::ex2(sc[0][1] - mu);
        const float p10 = ptx::ex2(sc[1][0] - mu), p11 = ptx::ex2(sc[1][1] - mu);
        l0 = l0 * alpha + (p00 + p01) + (p10 + p11);
        m0 = mn;
        pa[0] = ptx::pack_bf16x2(p00, p01);
        pa[2] = ptx::pack_bf16x2(p10, p11);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[nt][0] *= alpha;
          o[nt][1] *= alpha;
        }
      }
      if (HI) {
        float mx = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m1, mx);
        const float mu = (mn == -INFINITY) ? 0.f : mn;
        const float alpha = ptx::ex2(m1 - mu);
        const float p02 = ptx::ex2(sc[0][2] - mu), p03 = ptx::ex2(sc[0][3] - mu);
        const float p12 = ptx::ex2(sc[1][2] - mu), p13 = ptx::ex2(sc[1][3] - mu);
        l1 = l1 * alpha + (p02 + p03) + (p12 + p13);
        m1 = mn;
        pa[1] = ptx::pack_bf16x2(p02, p03);
        pa[3] = ptx::pack_bf16x2(p12, p13);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[nt][2] *= alpha;
          o[nt][3] *= alpha;
        }
      } else {
        pa[1] = 0u;
        pa[3] = 0u;
      }

      // O += P V.  Slots past the sequence end may hold any bits (NaN included):
      // their V words are zeroed in registers so 0 * NaN never reaches O.
      {
        uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
        if (nvalid < kChunk) {
          const int t0 = 2 * q4, t1 = 8 + 2 * q4;
          vm0 = (t0 < nvalid ? 0x0000ffffu : 0u) | (t0 + 1 < nvalid ? 0xffff0000u : 0u);
          vm1 = (t1 < nvalid ? 0x0000ffffu : 0u) | (t1 + 1 < nvalid ? 0xffff0000u : 0u);
        }
        const int tok = (((lane >> 3) & 1) << 3) + (lane & 7);
        const int sub = lane >> 4;
#pragma unroll
        for (int dt = 0; dt < KS; ++dt) {
          uint32_t b0, b1, b2, b3;
          ptx::ldmatrix_x4_trans(vb + sw128(tok, 2 * dt + sub), b0, b1, b2, b3);
          ptx::mma_bf16_16816(o[2 * dt], pa, b0 & vm0, b1 & vm1);
          ptx::mma_bf16_16816(o[2 * dt + 1], pa, b2 & vm0, b3 & vm1);
        }
      }
    }
    __syncwarp();
    if (issued < total) issue(stage);  // refill the stage just consumed

    // ------------------------------------------------------------ end of a piece?
    const bool seg_end = (cc.c + 1 == cc.nchunks);
    if (seg_end || i + 1 == total) {
      const bool sole = (piece_c0 == 0) && seg_end;
      float lt0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
      lt0 += __shfl_xor_sync(0xffffffffu, lt0, 2);
      float lt1 = 0.f;
      if (HI) {
        lt1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
        lt1 += __shfl_xor_sync(0xffffffffu, lt1, 2);
      }
      const int kvh = cc.seg / p.n_ht;
      const int ht = cc.seg % p.n_ht;
      const int head0 = kvh * p.group + ht * kHeadTile;
      const bool v0 = r0 < nrows, v1 = HI && (r0 + 8 < nrows);
      if (sole) {
        const float i0 = lt0 > 0.f ? 1.f / lt0 : 0.f;
        const float i1 = lt1 > 0.f ? 1.f / lt1 : 0.f;
        uint32_t* out0 = reinterpret_cast<uint32_t*>(
            p.out + (static_cast<int64_t>(cc.b) * p.num_heads + head0 + r0) * D);
        uint32_t* out1 = reinterpret_cast<uint32_t*>(
            p.out + (static_cast<int64_t>(cc.b) * p.num_heads + head0 + r0 + 8) * D);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int col2 = (nt * 8 + 2 * q4) / 2;
          if (v0) out0[col2] = ptx::pack_bf16x2(o[nt][0] * i0, o[nt][1] * i0);
          if (v1) out1[col2] = ptx::pack_bf16x2(o[nt][2] * i1, o[nt][3] * i1);
        }
      } else {
        const int64_t Ps = piece_x - piece_c0;  // linear index of the segment's chunk 0
        const int slot = static_cast<int>(w * 2 + (first_seg && Ps <= x0 ? 0 : 1));
        float* po = p.part_o + static_cast<int64_t>(slot) * kHeadTile * D;
        float* pml = p.part_ml + static_cast<int64_t>(slot) * kHeadTile * 2;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int col = nt * 8 + 2 * q4;
          if (v0) *reinterpret_cast<float2*>(po + r0 * D + col) = make_float2(o[nt][0], o[nt][1]);
          if (v1) *reinterpret_cast<float2*>(po + (r0 + 8) * D + col) = make_float2(o[nt][2], o[nt][3]);
        }
        if (q4 == 0) {
          if (v0) *reinterpret_cast<float2*>(pml + r0 * 2) = make_float2(m0, lt0);
          if (v1) *reinterpret_cast<float2*>(pml + (r0 + 8) * 2) = make_float2(m1, lt1);
        }
        __threadfence();
        __syncwarp();
        const int64_t segid = static_cast<int64_t>(cc.b) * segs + cc.seg;
        int prev = 0;
        if (lane == 0) prev = atomicAdd(p.counters + segid, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        const int64_t wf = worker_of(Ps, T, W);
        const int64_t wl = worker_of(Ps + cc.nchunks - 1, T, W);
        if (prev == static_cast<int>(wl - wf)) {
          // Last piece in: merge every piece of the segment.
          __threadfence();
          constexpr int CPL = D / 32;  // columns per lane
          float acc[kHeadTile][CPL];
          float M[kHeadTile], Ls[kHeadTile];
#pragma unroll
          for (int r = 0; r < kHeadTile; ++r) {
            M[r] = -INFINITY;
            Ls[r] = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) acc[r][j] = 0.f;
          }
          for (int64_t ww = wf; ww <= wl; ++ww) {
            const int sl = static_cast<int>(ww * 2 + (Ps <= worker_start(ww, T, W) ? 0 : 1));
            const float* qo = p.part_o + static_cast<int64_t>(sl) * kHeadTile * D + lane * CPL;
            const float* qml = p.part_ml + static_cast<int64_t>(sl) * kHeadTile * 2;
#pragma unroll
            for (int r = 0; r < kHeadTile; ++r) {
              if (r < nrows) {
                const float2 ml = __ldcg(reinterpret_cast<const float2*>(qml + r * 2));
                float ov[CPL];
                if constexpr (CPL == 4) {
                  const float4 t = __ldcg(reinterpret_cast<const float4*>(qo + r * D));
                  ov[0] = t.x; ov[1] = t.y; ov[2] = t.z; ov[3] = t.w;
                } else {
                  const float2 t = __ldcg(reinterpret_cast<const float2*>(qo + r * D));
                  ov[0] = t.x; ov[1] = t.y;
                }
                const float mn = fmaxf(M[r], ml.x);
                const float mu = (mn == -INFINITY) ? 0.f : mn;
                const float a = ptx::ex2(M[r] - mu), bw = ptx::ex2(ml.x - mu);
                Ls[r] = Ls[r] * a + ml.y * bw;
#pragma unroll
                for (int j = 0; j < CPL; ++j) acc[r][j] = acc[r][j] * a + ov[j] * bw;
                M[r] = mn;
              }
            }
          }
#pragma unroll
          for (int r = 0; r < kHeadTile; ++r) {
            if (r < nrows) {
              const float inv = Ls[r] > 0.f ? 1.f / Ls[r] : 0.f;
              uint16_t* dst = p.out + (static_cast<int64_t>(cc.b) * p.num_heads + head0 + r) * D + lane * CPL;
              if constexpr (CPL == 4) {
                uint2 v;
                v.x = ptx::pack_bf16x2(acc[r][0] * inv, acc[r][1] * inv);
                v.y = ptx::pack_bf16x2(acc[r][2] * inv, acc[r][3] * inv);
                *reinterpret_cast<uint2*>(dst) = v;
              } else {
                *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[r][0] * inv, acc[r][1] * inv);
              }
            }
          }
          if (lane == 0) p.counters[segid] = 0;
        }
      }
      first_seg = false;
      if (i + 1 < total) {
        cursor_next(cc, p, segs, cap);
        load_q(cc);
        piece_x = x0 + i + 1;
        piece_c0 = 0;
      }
    } else {
      ++cc.c;
    }
  }
}

// ------------------------------------------------------------------ host side
namespace {
constexpr int kWarps = 4;
constexpr int kStages128 = 3;
constexpr int kStages64 = 6;

template <int D, int STAGES>
constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(kWarps) * STAGES * Geo<D>::kStageBytes +
         static_cast<size_t>(kWarps) * STAGES * 8;
}

template <int D, int STAGES, bool HI>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                     int grid, cudaStream_t stream) {
  auto kern = decode_split_kernel<D, kWarps, STAGES, HI>;
  constexpr size_t smem = smem_bytes<D, STAGES>();
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  kern<<<grid, kWarps * 32, smem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}
}  // namespace

DecodeLaunch decode_launch_config(int head_dim, int group) {
  (void)group;
  DecodeLaunch l;
  l.warps_per_cta = kWarps;
  l.ctas_per_sm = 2;
  l.smem_bytes = head_dim == 64 ? smem_bytes<64, kStages64>() : smem_bytes<128, kStages128>();
  return l;
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                          int grid, cudaStream_t stream) {
  const bool hi = p.group > 8;
  if (p.head_dim == 64)
    return hi ? launch_t<64, kStages64, true>(p, tk, tv, grid, stream)
              : launch_t<64, kStages64, false>(p, tk, tv, grid, stream);
  return hi ? launch_t<128, kStages128, true>(p, tk, tv, grid, stream)
            : launch_t<128, kStages128, false>(p, tk, tv, grid, stream);
}

}  // namespace gqa
