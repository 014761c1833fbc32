// Paged GQA/MQA decode attention: one new query token per sequence.
//
// What is computed (page "TensorRT对Multi-Query Attention的专项优化支持": decode re-reads
// all cached K/V; MQA/GQA query heads share K/V heads and the plugin avoids copying or
// broadcasting K/V to them; QK^T then AV on tensor cores with tiled shared-memory K/V
// prefetch; paged cache.  tiny-llm "优化" page: GQA, block table + gather,
// FlashDecoding for long contexts):
//
//   out[b, h] = sum_t softmax_t(scale * q[b, h] . K_b[t, kvh]) V_b[t, kvh],  kvh = h / G.
//
// Design (B200, sm_100a), one CTA per SM:
//   * Work list.  The context of every (sequence b, segment s = kv head x head tile) is
//     cut into 64-token blocks; all blocks of all segments form one linear list in
//     (b, s, block) order, split into equal contiguous ranges, one per CTA (split-KV /
//     FlashDecoding, balanced at block granularity whatever the length mix).  Each CTA
//     derives its range from seq_lens in a short prologue: no planning kernel and no
//     host synchronisation.
//   * Producer warp.  Walks the CTA's blocks, reads page ids from the block table
//     through a prefetched register window and issues one 3-D TMA copy per 16-token
//     sub-chunk and tensor (box: 64 columns x 16 rows x head_dim/64 column groups,
//     128-byte swizzle) into a ring of 64-token stages (full/empty mbarriers).  It also
//     writes a small descriptor per stage.
//   * Consumer warps (mma.sync m16n8k16, bf16 in, fp32 accumulate), tokens on the M side:
//     S^T = K Q^T, softmax down the token axis, P^T moved to B-fragment layout with
//     movmatrix, O^T += V^T P^T with V^T read by ldmatrix.trans.  Every K/V row in shared
//     memory serves all query heads of its kv head, so HBM is read once per kv head.
//     Each of the 4 consumers takes one 16-token sub-chunk of every stage for all rows of
//     the segment (up to 16: a group of heads, or several query tokens' groups); at a
//     piece end their partial softmax states are combined in shared memory by an
//     epilogue warp.  More rows per kv head run on the tcgen05 kernel (decode_tc.cu).
//   * Online softmax in the log2 domain with a lazily moved reference: O and the sum are
//     rescaled only when a head's running maximum rises by more than 8 (factor 256);
//     numerator and denominator share the reference, so the result is unchanged.
//   * Cross-CTA merge.  A segment spanning several CTAs leaves one piece per CTA
//     (unnormalised O, reference max, sum); the last CTA to finish its piece (arrival
//     counter) merges all pieces with their log-sum-exp weights in its epilogue warp,
//     writes out, and resets the counter to zero.
//   * Safety.  Page ids and lengths are range-checked on the device (bad work is skipped
//     and an error bit set); every mbarrier wait is bounded in time.
#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

namespace {

// F8: the cache holds e4m3 codes (one byte per element) instead of bf16.
template <int D, bool F8 = false>
struct Geo {
  static constexpr int kElem = F8 ? 1 : 2;
  static constexpr int kBoxes = D / 64;                      // bf16: 64-column (128-byte) boxes
  static constexpr int kBoxBytes = kChunk * 128;             // bf16: 16 rows x 128 bytes
  static constexpr int kSubBytes = kChunk * D * kElem;       // one 16-token K (or V) tile
  // A stage: for each of the 4 sub-chunks its K and V tiles, adjacent
  static constexpr int kStageBytes = 2 * kSubChunks * kSubBytes;
  // Query heads whose fp32 partial O (D floats each) fit one sub-chunk tile: a consumer
  // hands its partial to the epilogue in its own K and V sub-chunk tiles.
  static constexpr int kHeadsPerSub = kSubBytes / (4 * D);
};

constexpr float kRescaleThreshold = 8.0f;
constexpr int kMaxWarps = 9;

// Per-stage descriptor, written by the producer before the stage's full barrier
// completes (release/acquire through the mbarrier).
struct StageInfo {
  int64_t seg_base;  // linear index of block 0 of this block's segment
  int b, seg, blk, nblk;
  int nvalid;        // valid tokens of this block (1..64)
  int submask;       // bit s: sub-chunk s was loaded
  int flags;
  int rem;           // tokens of the sequence from this block's first one on (unclamped)
};
enum : int { kFirstOfPiece = 1, kLastOfPiece = 2, kSole = 4, kFirstPieceOfCta = 8 };

__device__ __forceinline__ int eff_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

struct Cursor {
  int b;     // sequence
  int seg;   // kv_head * n_ht + head_tile
  int kvh;   // seg / n_ht
  int ht;    // seg % n_ht
  int blk;   // block within the segment
  int nblk;  // blocks per segment of sequence b
  int len;   // effective context length of sequence b
};

__device__ __forceinline__ void cursor_load_seq(Cursor& cu, const DecodeParams& p, int cap) {
  cu.len = (cu.b >= 0 && cu.b < p.num_seqs) ? eff_len(__ldg(p.seq_lens + cu.b), cap) : 0;
  cu.nblk = (cu.len + kBlock - 1) / kBlock;
}

// Step a cursor to the next block of the work list (only while blocks remain).
// next_len holds seq_lens[c.b + 1], loaded ahead of the cursor reaching it.
__device__ __forceinline__ void walk_next(Cursor& c, int& next_len, const DecodeParams& p, int segs,
                                          int cap) {
  if (++c.blk < c.nblk) return;
  c.blk = 0;
  if (++c.seg < segs) {
    if (++c.ht == p.n_ht) {
      c.ht = 0;
      ++c.kvh;
    }
    return;
  }
  c.seg = c.kvh = c.ht = 0;
  do {
    ++c.b;
    c.len = (c.b < p.num_seqs) ? eff_len(next_len, cap) : 0;
    c.nblk = (c.len + kBlock - 1) / kBlock;
    next_len = (c.b + 1 < p.num_seqs) ? __ldg(p.seq_lens + c.b + 1) : 0;
  } while (c.nblk == 0 && c.b + 1 < p.num_seqs);
}

__device__ __forceinline__ int64_t worker_start(int64_t w, int64_t T, int64_t W) { return w * T / W; }
// The worker (CTA) whose range holds linear block x.
__device__ __forceinline__ int64_t worker_of(int64_t x, int64_t T, int64_t W) {
  return ((x + 1) * W - 1) / T;
}
__device__ __forceinline__ int piece_slot(int64_t w, int64_t seg_base, int64_t T, int64_t W) {
  return static_cast<int>(w * 2 + (seg_base <= worker_start(w, T, W) ? 0 : 1));
}

// One 16-token sub-chunk for NT n-tiles of 8 heads: S^T = K Q^T, online softmax down the
// token axis, O^T += V^T P^T.  kb/vb: shared addresses of the sub-chunk's swizzled K/V.
// MQ (several query tokens per sequence): column (head) e of n-tile nt sees only the
// first rem - cdrop[nt][e] tokens from this sub-chunk's first one (rem: tokens of the
// sequence from there on; cdrop: newer query tokens than the column's own).
template <int D, int NT, bool MQ>
__device__ __forceinline__ void attend_subchunk(uint32_t kb, uint32_t vb, int nvalid,
                                                const uint32_t (&kofs)[4], const uint32_t (&vofs)[4],
                                                const uint32_t (&qf)[D / 16][NT][2],
                                                float (&o)[D / 16][NT][4], float (&mref)[NT][2],
                                                float (&lsum)[NT][2], float sl2, int g, int q,
                                                int rem, int max_drop, const int (&cdrop)[NT][2]) {
  using G_ = Geo<D>;
  constexpr int KS = D / 16;
  constexpr int MT = D / 16;
  float s[2][NT][4];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[c][nt][0] = s[c][nt][1] = s[c][nt][2] = s[c][nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a[4];
    ptx::ldmatrix_x4(kb + (ks >> 2) * G_::kBoxBytes + kofs[ks & 3], a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) ptx::mma_bf16_16816(s[ks & 1][nt], a, qf[ks][nt][0], qf[ks][nt][1]);
  }
  // c0,c1: token g, heads 2q, 2q+1;  c2,c3: token g + 8.
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[nt][e] = (s[0][nt][e] + s[1][nt][e]) * sl2;
  if constexpr (MQ) {
    if (rem - max_drop < kChunk) {  // a column's window may end inside this sub-chunk
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int lim = rem - cdrop[nt][e];
          if (g >= lim) sc[nt][e] = -INFINITY;
          if (g + 8 >= lim) sc[nt][e + 2] = -INFINITY;
        }
    }
  } else if (nvalid < kChunk) {
    const bool v0 = g < nvalid, v1 = g + 8 < nvalid;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (!v0) sc[nt][0] = sc[nt][1] = -INFINITY;
      if (!v1) sc[nt][2] = sc[nt][3] = -INFINITY;
    }
  }
  float mx[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float m = fmaxf(sc[nt][e], sc[nt][e + 2]);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      mx[nt][e] = m;
    }
  bool need = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) need |= mx[nt][e] > mref[nt][e] + kRescaleThreshold;
  if (__any_sync(0xffffffffu, need)) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float mn = fmaxf(mref[nt][e], mx[nt][e]);
        const float alpha = (mn == mref[nt][e]) ? 1.f : ptx::ex2(mref[nt][e] - mn);
        mref[nt][e] = mn;
        lsum[nt][e] *= alpha;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][nt][e] *= alpha;
          o[mt][nt][e + 2] *= alpha;
        }
      }
  }
  uint32_t pb[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float mu0 = (mref[nt][0] == -INFINITY) ? 0.f : mref[nt][0];
    const float mu1 = (mref[nt][1] == -INFINITY) ? 0.f : mref[nt][1];
    const float p0 = ptx::ex2(sc[nt][0] - mu0), p1 = ptx::ex2(sc[nt][1] - mu1);
    const float p2 = ptx::ex2(sc[nt][2] - mu0), p3 = ptx::ex2(sc[nt][3] - mu1);
    lsum[nt][0] += p0 + p2;
    lsum[nt][1] += p1 + p3;
    pb[nt][0] = ptx::movmatrix_trans(ptx::pack_bf16x2(p0, p1));  // tokens 2q, 2q+1 of head g
    pb[nt][1] = ptx::movmatrix_trans(ptx::pack_bf16x2(p2, p3));  // tokens 8 + 2q ..
  }
  // Slots past the sequence end may hold any bits (NaN included): their V words are
  // zeroed in registers so 0 * NaN never reaches O.
  uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
  if (nvalid < kChunk) {
    const int t0 = 2 * q, t1 = 8 + 2 * q;
    vm0 = (t0 < nvalid ? 0x0000ffffu : 0u) | (t0 + 1 < nvalid ? 0xffff0000u : 0u);
    vm1 = (t1 < nvalid ? 0x0000ffffu : 0u) | (t1 + 1 < nvalid ? 0xffff0000u : 0u);
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    uint32_t a[4];
    ptx::ldmatrix_x4_trans(vb + (mt >> 2) * G_::kBoxBytes + vofs[mt & 3], a[0], a[1], a[2], a[3]);
    a[0] &= vm0;
    a[1] &= vm0;
    a[2] &= vm1;
    a[3] &= vm1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) ptx::mma_bf16_16816(o[mt][nt], a, pb[nt][0], pb[nt][1]);
  }
}

// The same sub-chunk over an e4m3 cache, on fp16 MMAs (e4m3 -> fp16 is exact; q is
// converted to fp16 when its fragments are loaded, P is packed as fp16).  K: one 16-byte
// ldmatrix row is 16 head-dim values of one token, so thread (g, q) receives values
// 4q .. 4q + 3 of a 16-value chunk, and the contraction over head_dim uses that order
// (the q fragments follow it).  V^T comes from the transposing byte ldmatrix (16 x 16
// codes per matrix), whose lane (g, q) receives tokens 2q, 2q+1, 2q+8, 2q+9 of dims g and
// g + 8: widened, that is the mma A fragment of V^T as it stands (1.8-3.1 % faster than
// widening row-major codes and transposing each pair with movmatrix; the transposing
// 16-bit ldmatrix with one byte permute per register measured slower than both).
template <int D, int NT>
__device__ __forceinline__ void attend_subchunk_f8(uint32_t kb, uint32_t vb, int nvalid,
                                                   const uint32_t (&ofs)[D / 32], const uint32_t (&vofs)[D / 32],
                                                   const uint32_t (&qf)[D / 16][NT][2],
                                                   float (&o)[D / 16][NT][4], float (&mref)[NT][2],
                                                   float (&lsum)[NT][2], float sl2, int g, int q) {
  constexpr int MT = D / 16;
  float s[2][NT][4];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[c][nt][0] = s[c][nt][1] = s[c][nt][2] = s[c][nt][3] = 0.f;
#pragma unroll
  for (int kx = 0; kx < D / 32; ++kx) {
    uint32_t r[4];
    ptx::ldmatrix_x4(kb + ofs[kx], r[0], r[1], r[2], r[3]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // k-step 2 kx + h: chunk 2 kx + h (r[2h]: token g, r[2h+1]: g + 8)
      const uint32_t a[4] = {ptx::e4m3x2_lo(r[2 * h]), ptx::e4m3x2_lo(r[2 * h + 1]), ptx::e4m3x2_hi(r[2 * h]),
                             ptx::e4m3x2_hi(r[2 * h + 1])};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) ptx::mma_f16_16816(s[h][nt], a, qf[2 * kx + h][nt][0], qf[2 * kx + h][nt][1]);
    }
  }
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[nt][e] = (s[0][nt][e] + s[1][nt][e]) * sl2;
  if (nvalid < kChunk) {
    const bool v0 = g < nvalid, v1 = g + 8 < nvalid;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (!v0) sc[nt][0] = sc[nt][1] = -INFINITY;
      if (!v1) sc[nt][2] = sc[nt][3] = -INFINITY;
    }
  }
  float mx[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float m = fmaxf(sc[nt][e], sc[nt][e + 2]);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      mx[nt][e] = m;
    }
  bool need = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) need |= mx[nt][e] > mref[nt][e] + kRescaleThreshold;
  if (__any_sync(0xffffffffu, need)) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float mn = fmaxf(mref[nt][e], mx[nt][e]);
        const float alpha = (mn == mref[nt][e]) ? 1.f : ptx::ex2(mref[nt][e] - mn);
        mref[nt][e] = mn;
        lsum[nt][e] *= alpha;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][nt][e] *= alpha;
          o[mt][nt][e + 2] *= alpha;
        }
      }
  }
  uint32_t pb[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float mu0 = (mref[nt][0] == -INFINITY) ? 0.f : mref[nt][0];
    const float mu1 = (mref[nt][1] == -INFINITY) ? 0.f : mref[nt][1];
    const float p0 = ptx::ex2(sc[nt][0] - mu0), p1 = ptx::ex2(sc[nt][1] - mu1);
    const float p2 = ptx::ex2(sc[nt][2] - mu0), p3 = ptx::ex2(sc[nt][3] - mu1);
    lsum[nt][0] += p0 + p2;
    lsum[nt][1] += p1 + p3;
    pb[nt][0] = ptx::movmatrix_trans(ptx::pack_f16x2(p0, p1));
    pb[nt][1] = ptx::movmatrix_trans(ptx::pack_f16x2(p2, p3));
  }
  // Codes past the sequence end may be anything (NaN included): zeroed after conversion.
  uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
  if (nvalid < kChunk) {
    const int t0 = 2 * q, t1 = 8 + 2 * q;
    vm0 = (t0 < nvalid ? 0x0000ffffu : 0u) | (t0 + 1 < nvalid ? 0xffff0000u : 0u);
    vm1 = (t1 < nvalid ? 0x0000ffffu : 0u) | (t1 + 1 < nvalid ? 0xffff0000u : 0u);
  }
#pragma unroll
  for (int vx = 0; vx < D / 32; ++vx) {
    uint32_t r[4];
    // V^T straight from the transposing byte ldmatrix: r[2h] holds dim 16(2vx+h) + g and
    // r[2h+1] dim 16(2vx+h) + g + 8, tokens 2q, 2q+1, 2q+8, 2q+9 in bytes 0..3
    ptx::ldmatrix_m16n16_x2_trans_b8(vb + vofs[vx], r[0], r[1], r[2], r[3]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // O^T tile mt = 2 vx + h
      uint32_t a[4];
      a[0] = ptx::e4m3x2_lo(r[2 * h]) & vm0;      // dim g, tokens 2q, 2q+1
      a[1] = ptx::e4m3x2_lo(r[2 * h + 1]) & vm0;  // dim g + 8
      a[2] = ptx::e4m3x2_hi(r[2 * h]) & vm1;      // dim g, tokens 2q+8, 2q+9
      a[3] = ptx::e4m3x2_hi(r[2 * h + 1]) & vm1;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) ptx::mma_f16_16816(o[2 * vx + h][nt], a, pb[nt][0], pb[nt][1]);
    }
  }
}

}  // namespace

// Launch shape: CTAs per SM (several producer warps per SM keep more TMA copies in
// flight) and the per-SM shared-memory budget shared by their rings and merge areas
// (overridable at compile time for tuning sweeps).
#ifndef GQA_CTAS_TOKEN_SPLIT
#define GQA_CTAS_TOKEN_SPLIT 2
#endif
#ifndef GQA_SMEM_PER_SM_KB
#define GQA_SMEM_PER_SM_KB 220
#endif

constexpr int kWsCtasPerSm = GQA_CTAS_TOKEN_SPLIT;
// The 8-bit cache moves half the bytes per stage; its launch shape is set on its own.
// With one copy per sub-chunk for K and V and multiply-shift page arithmetic in the
// producer, two CTAs per SM (5 stages each) measure faster than three (3 stages, 96
// registers, spills): 36.2 against 41.5 us on the GQA serving batch, 204 against 215 us
// on the long-context batch, 284.5 against 281.5 us on the continuous batch.  (Before
// those producer changes three CTAs were the faster shape.)
#ifndef GQA_F8_CTAS
#define GQA_F8_CTAS 2
#endif
#ifndef GQA_F8_SMEM_PER_SM_KB
#define GQA_F8_SMEM_PER_SM_KB 212
#endif
constexpr int kWsCtasPerSmF8 = GQA_F8_CTAS;

// D: head_dim.  NT: 8-head n-tiles per consumer (each consumer takes one 16-token
// sub-chunk of every stage for all rows).  C: consumer warps.  S: stages.  MQ:
// several query tokens per sequence (p.q_len): a kv head's rows are its group of heads
// for each query token in turn (row r: token r / group, head r % group), one segment.
// F8: the cache holds e4m3 codes with one scale per kv head for K and for V
// (p.k_scales, p.v_scales); the K scale joins the score scale of a piece, the V scale
// the output of its combine.
template <int D, int NT, int C, int S, bool MQ, bool F8>
__global__ void __launch_bounds__((C + 2) * 32, F8 ? kWsCtasPerSmF8 : kWsCtasPerSm)
decode_ws_kernel(const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using G_ = Geo<D, F8>;
  constexpr int MT = D / 16;
  constexpr int NH = 8 * NT;             // heads one consumer covers
  constexpr int HS = G_::kHeadsPerSub;   // partial rows that fit one sub-chunk tile
  static_assert(C == kSubChunks, "one consumer per sub-chunk");
  static_assert(NH <= 2 * HS, "a consumer's partial must fit its K and V sub-chunk tiles");
  static_assert(!(F8 && MQ), "the 8-bit cache serves one query token per sequence");

  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_wtot[kMaxWarps];
  __shared__ int s_start_b;
  __shared__ int64_t s_start_base;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int B = p.num_seqs;
  const int segs = p.num_kv_heads * p.n_ht;
  const int cap = p.max_blocks * p.page_size;
  // Rows per kv head, and the memory row (of q and out) of row r of kv head kvh.
  const int grp = MQ ? p.group * p.q_len : p.group;
  auto seq_row = [&](int b, int kvh, int r) -> int64_t {
    if constexpr (MQ) {
      const int i = r / p.group;
      return (static_cast<int64_t>(b) * p.q_len + i) * p.num_heads + kvh * p.group + (r - i * p.group);
    } else {
      return static_cast<int64_t>(b) * p.num_heads + kvh * p.group + r;
    }
  };
  const int rows_per_seq = MQ ? p.num_heads * p.q_len : p.num_heads;

  // ---------------------------------------------------------------- prologue
  // Pass 1: block counts per sequence, their total T (and zero rows of empty sequences).
  int64_t n_first = 0;  // this thread's count in the first tile of sequences
  int64_t mine = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = __ldg(p.seq_lens + b);
    const int Le = eff_len(L, cap);
    if ((L < 0 || L > cap) && blockIdx.x == 0) atomicOr(p.err, kErrBounds);
    if (Le == 0 && (b % gridDim.x) == blockIdx.x) {
      uint32_t* o = reinterpret_cast<uint32_t*>(p.out + static_cast<int64_t>(b) * rows_per_seq * D);
      for (int i = 0; i < rows_per_seq * D / 2; ++i) o[i] = 0u;
    }
    const int64_t n = static_cast<int64_t>((Le + kBlock - 1) / kBlock) * segs;
    if (b == static_cast<int>(threadIdx.x)) n_first = n;
    mine += n;
  }
  if (threadIdx.x == 0) s_start_b = -1;
  // Inclusive block-wide scan of one value per thread; returns (inclusive, tile total).
  auto block_scan = [&](int64_t n, int64_t& tot) -> int64_t {
    int64_t incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) s_wtot[warp] = incl;
    __syncthreads();
    int64_t pre = 0;
    tot = 0;
    for (int i = 0; i < nwarps; ++i) {
      if (i < warp) pre += s_wtot[i];
      tot += s_wtot[i];
    }
    __syncthreads();  // s_wtot is reused by the next scan
    return incl + pre;
  };
  int64_t T = 0, W = 0, x0 = 0, x1 = 0;
  const int64_t w = blockIdx.x;
  if (B <= static_cast<int>(blockDim.x)) {
    // One tile holds every sequence: the scan gives T and the start in one pass.
    const int64_t incl = block_scan(n_first, T);
    // Only the first T CTAs get work when there are fewer blocks than CTAs, so every
    // CTA in use owns at least one block and a segment's pieces come from exactly the
    // CTAs worker_of(first block) .. worker_of(last block).
    W = min(static_cast<int64_t>(p.num_workers), T);
    if (w >= W) return;  // (also covers T == 0)
    x0 = worker_start(w, T, W);
    x1 = worker_start(w + 1, T, W);
    if (n_first > 0 && x0 >= incl - n_first && x0 < incl) {
      s_start_b = threadIdx.x;
      s_start_base = incl - n_first;
    }
    __syncthreads();
  } else {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
    if (lane == 0) s_wtot[warp] = mine;
    __syncthreads();
    for (int i = 0; i < nwarps; ++i) T += s_wtot[i];
    W = min(static_cast<int64_t>(p.num_workers), T);
    if (w >= W) return;
    x0 = worker_start(w, T, W);
    x1 = worker_start(w + 1, T, W);
    __syncthreads();  // s_wtot is reused below
    // Pass 2: locate the sequence holding block x0 (tiled block scan).
    int64_t base = 0;
    for (int t0 = 0; t0 < B && base <= x0; t0 += blockDim.x) {
      const int b = t0 + threadIdx.x;
      int64_t n = 0;
      if (b < B) n = static_cast<int64_t>((eff_len(__ldg(p.seq_lens + b), cap) + kBlock - 1) / kBlock) * segs;
      int64_t tot = 0;
      const int64_t incl = base + block_scan(n, tot);
      if (n > 0 && x0 >= incl - n && x0 < incl) {
        s_start_b = b;
        s_start_base = incl - n;
      }
      base += tot;
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- shared layout
  const uint32_t smem0 = ptx::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (smem0 & 1023u)) & 1023u;
  uint8_t* base_ptr = smem_raw + pad;
  const uint32_t ring = smem0 + pad;
  // Token split: at a piece end each consumer leaves its partial O^T in the part of the
  // stage only it read (its sub-chunk's K tile, and V tile for a second n-tile) and its
  // (max, sum) pairs in cml[stage]; the epilogue warp combines them and releases the stage.
  constexpr int kCml = S * C * NH * 2;  // floats
  float* cml = reinterpret_cast<float*>(base_ptr + S * G_::kStageBytes);
  // Token split: the query rows of a piece arrive with its first block (bulk copy).
  constexpr int kQBytes = NH * D * 2;
  uint8_t* qbuf = reinterpret_cast<uint8_t*>(cml + kCml);
  StageInfo* info = reinterpret_cast<StageInfo*>(qbuf + S * kQBytes);
  const uint32_t full_bar = ptx::smem_u32(info + S);
  const uint32_t empty_bar = full_bar + 8 * S;
  const uint32_t comb_bar = empty_bar + 8 * S;  // token split: consumers -> epilogue
  // The epilogue's merged partial of the other pieces of its final segment: [8][D] O then
  // [8] (max, sum) pairs.
  float* pre_o = reinterpret_cast<float*>(base_ptr + ((reinterpret_cast<uintptr_t>(info + S) + 24 * S + 15 -
                                                       reinterpret_cast<uintptr_t>(base_ptr)) & ~uintptr_t{15}));
  float* pre_ml = pre_o + 8 * D;

  const int start_b = s_start_b;
  const int64_t start_base = s_start_base;
  if (start_b < 0) {  // cannot happen for a non-empty range; never index with it
    if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar + 8 * s, 1);
      ptx::mbar_init(empty_bar + 8 * s, C);
      ptx::mbar_init(comb_bar + 8 * s, C);
    }
    ptx::fence_mbarrier_init();
  }
  __syncthreads();

  const int64_t total = x1 - x0;
  const uint64_t limit = p.wait_limit_ns;

  Cursor cu;
  cu.b = start_b;
  cursor_load_seq(cu, p, cap);
  {
    const int64_t off = x0 - start_base;
    cu.seg = static_cast<int>(off / cu.nblk);
    cu.blk = static_cast<int>(off % cu.nblk);
    cu.kvh = cu.seg / p.n_ht;
    cu.ht = cu.seg - cu.kvh * p.n_ht;
  }

  if (warp == C) {
    // ============================================================ producer warp
    if (lane == 0) {
      ptx::prefetch_tensormap(&tmap_k);
      ptx::prefetch_tensormap(&tmap_v);
    }
    const uint64_t policy = ptx::policy_evict_first();
    // Block-table rows are read 32 entries at a time (one per lane) into a register
    // window, with the window needed next already in flight, so no TMA issue waits on
    // a dependent global load.  Lanes s and s + 4 (s < 4) look up sub-chunk s of every
    // block; lane s owns its copy.
    const int ps = p.page_size;
    const uint32_t pm = p.ps_magic;
    const int psh = p.ps_shift;
    auto load_window = [&](int b, int k) -> int {
      const int e = 32 * k + lane;
      return (b >= 0 && b < B && e < p.max_blocks)
                 ? __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + e) : -1;
    };
    int wb = -1, wk = -1, wval = -1;  // window in use: row wb, entries [32 wk, 32 wk + 32)
    int nb = -1, nk = -1, nval = -1;  // window prefetched next
    // length of the sequence after cu.b, loaded ahead of the cursor reaching it
    int next_len = (cu.b + 1 < B) ? __ldg(p.seq_lens + cu.b + 1) : 0;
    auto prefetch_after = [&](const Cursor& c, int k) {
      const int entries = c.len > 0 ? fast_div(c.len - 1, pm, psh) + 1 : 0;
      if (32 * (k + 1) < entries) { nb = c.b; nk = k + 1; }
      else if (c.seg + 1 < segs) { nb = c.b; nk = 0; }
      else { nb = c.b + 1; nk = 0; }
      nval = load_window(nb, nk);
    };
    // The page of this lane's sub-chunk (lanes < 8; -1 past the sequence's end) and the
    // sub-chunk's first token within it (toff).
    auto page_of = [&](const Cursor& c, int& toff) -> int {
      const int e0 = fast_div(c.blk * kBlock, pm, psh);
      const int k = e0 >> 5;
      if (c.b != wb || k != wk) {
        if (c.b == nb && k == nk) { wval = nval; }
        else { wval = load_window(c.b, k); }
        wb = c.b;
        wk = k;
        prefetch_after(c, k);
      }
      const int t = c.blk * kBlock + (lane & 3) * kChunk;
      const int e = fast_div(t, pm, psh);
      toff = t - e * ps;
      const int pg = __shfl_sync(0xffffffffu, wval, e - 32 * k);  // a block never straddles two windows
      return (lane < 2 * kSubChunks && t < c.len) ? pg : -1;
    };
    // Bytes of a piece's query rows (contiguous in q): the token split stages them.
    auto q_rows_bytes = [&](const Cursor& c) -> uint32_t {
      return static_cast<uint32_t>(min(NH, grp - c.ht * NH)) * D * 2u;
    };
    // Stage layout: sub-chunk s holds its K tile then its V tile (V then K when the
    // paired map's lower pool is V), each kSubBytes.
    const int pair = p.kv_pair;
    int toff = 0;
    int page = page_of(cu, toff);
    int stage = 0;
    uint32_t phase = 0;  // parity of the current pass over the ring
    int piece_blk0 = cu.blk;
    int64_t seg_base = x0 - cu.blk;
    for (int64_t i = 0; i < total; ++i) {
      if (i >= S) {
        const bool ok = ptx::mbar_wait_bounded(empty_bar + 8 * stage, phase ^ 1u, limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) atomicOr(p.err, kErrTimeout);
          // give copies still in flight a bounded chance to land, then leave
          for (int64_t j = i - S; j < i; ++j)
            ptx::mbar_wait_bounded(full_bar + 8 * (j % S), static_cast<uint32_t>((j / S) & 1), limit);
          return;
        }
      }
      const int nvalid = min(kBlock, cu.len - cu.blk * kBlock);
      const bool want = lane < kSubChunks && lane * kChunk < nvalid;  // (page >= 0 there)
      const bool ok = want && page >= 0 && page < p.num_pages;
      const uint32_t submask = __ballot_sync(0xffffffffu, ok) & 0xFu;
      if (__any_sync(0xffffffffu, want && !ok) && lane == 0) atomicOr(p.err, kErrBounds);
      const bool first = (i == 0) || cu.blk == 0;
      const bool last = (i + 1 == total) || (cu.blk + 1 == cu.nblk);
      if (first) piece_blk0 = cu.blk;
      if (lane == 0) {
        StageInfo& si = info[stage];
        si.seg_base = seg_base;
        si.b = cu.b;
        si.seg = cu.seg;
        si.blk = cu.blk;
        si.nblk = cu.nblk;
        si.nvalid = nvalid;
        si.submask = static_cast<int>(submask);
        si.rem = cu.len - cu.blk * kBlock;
        si.flags = (first ? kFirstOfPiece : 0) | (last ? kLastOfPiece : 0) |
                   ((last && piece_blk0 == 0 && cu.blk + 1 == cu.nblk) ? kSole : 0) |
                   (seg_base <= x0 ? kFirstPieceOfCta : 0);
        uint32_t bytes = static_cast<uint32_t>(__popc(submask)) * 2u * G_::kSubBytes;
        if (first && !p.arm_without_copy) bytes += q_rows_bytes(cu);
        if (bytes) ptx::mbar_arrive_expect_tx(full_bar + 8 * stage, bytes);
        else ptx::mbar_arrive(full_bar + 8 * stage);
      }
      if (i == 0) ptx::pdl_wait_prerequisites();  // K/V may still be written by the previous kernel
      __syncwarp();
      {
        if (first && !p.arm_without_copy) {
          const int kvh = cu.kvh, ht = cu.ht;
          if constexpr (MQ) {
            // One copy per query token (its group's rows are contiguous in q); a
            // segment is the whole kv head (ht == 0) when there are several tokens.
            for (int i = lane - 2 * kSubChunks; i >= 0 && i < p.q_len; i += 32 - 2 * kSubChunks)
              ptx::bulk_load(ptx::smem_u32(qbuf + stage * kQBytes) + i * p.group * D * 2,
                             p.q + seq_row(cu.b, kvh, i * p.group) * D,
                             static_cast<uint32_t>(p.group) * D * 2u, full_bar + 8 * stage);
          } else if (lane == 2 * kSubChunks) {
            ptx::bulk_load(ptx::smem_u32(qbuf + stage * kQBytes), p.q + seq_row(cu.b, kvh, ht * NH) * D,
                           q_rows_bytes(cu), full_bar + 8 * stage);
          }
        }
      }
      {
        const int sc = lane & (kSubChunks - 1);
        // first pool row of the sub-chunk (page, kv head, token); lanes s and s + 4 agree
        const int row = (page * p.num_kv_heads + cu.kvh) * ps + toff;
        const uint32_t dst = ring + stage * G_::kStageBytes + sc * 2 * G_::kSubBytes;
        const uint32_t bar = full_bar + 8 * stage;
        if (p.arm_without_copy) {
        } else if constexpr (!F8) {
          // bf16: lane l < 8 copies sub-chunk l % 4 of K (l < 4) or V (l >= 4), all head_dim/64
          // column boxes of the 16 rows in one copy (a warp issues tiled copies faster the
          // more of its lanes take part: 52.7 against 53.0 us on the GQA batch)
          if (lane < 2 * kSubChunks && ((submask >> sc) & 1u)) {
            const bool is_v = lane >= kSubChunks;
            ptx::tma_load_3d(dst + (is_v ? G_::kSubBytes : 0), is_v ? &tmap_v : &tmap_k, bar, 0, row, 0, policy);
          }
        } else if (ok) {
          // e4m3 codes, 128-byte rows (a sub-chunk is 16 * D / 128 of them): lane s < 4
          // copies sub-chunk s of both pools in one copy when they share a map, else of K
          // and of V apart (eight lanes measured slower: 248.4 against 241.7 us on the
          // long-context batch)
          if (pair != 0) {
            ptx::tma_load_3d(dst, &tmap_k, bar, 0, row / (128 / D), 0, policy);
          } else {
            ptx::tma_load_2d(dst, &tmap_k, bar, 0, row / (128 / D), policy);
            ptx::tma_load_2d(dst + G_::kSubBytes, &tmap_v, bar, 0, row / (128 / D), policy);
          }
        }
      }
      if (++stage == S) {
        stage = 0;
        phase ^= 1u;
      }
      if (i + 1 < total) {
        walk_next(cu, next_len, p, segs, cap);
        if (cu.blk == 0) seg_base = x0 + i + 1;
        page = page_of(cu, toff);
      }
    }
    return;
  }

  if (warp == C + 1) {
    // ============================================================ epilogue warp
    // Walks the same block list.  At each piece end it waits for the C consumers' states
    // in the stage, combines them, writes out (or this CTA's piece of the segment),
    // releases the stage to the producer, and runs the cross-CTA step; the consumers
    // meanwhile go on with the next blocks.
    constexpr int CPL = D / 32;  // columns per lane
    const int d0 = lane * CPL;
    const int hps = p.heads_per_seg;
    int next_len = (cu.b + 1 < B) ? __ldg(p.seq_lens + cu.b + 1) : 0;
    uint32_t comb_phase = 0;  // bit s: parity of the next completion of comb_bar[s]
    // Rows h0..h0+7 of every piece of a segment except worker skip's, merged (log-sum-exp
    // over the pieces' (max, sum) pairs); loads batched per piece.
    auto merge_pieces = [&](int64_t sbase, int64_t wf, int64_t wl, int64_t skip, int h0, int nrows,
                            float (&M)[8], float (&L)[8], float (&acc)[8][CPL]) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        M[k] = -INFINITY;
        L[k] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[k][c] = 0.f;
      }
      for (int64_t ww = wf; ww <= wl; ++ww) {
        if (ww == skip) continue;
        const int64_t sl = piece_slot(ww, sbase, T, W);
        float2 mlv[8];
        float v[8][CPL];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int h = min(h0 + k, nrows - 1);
          mlv[k] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (sl * hps + h) * 2));
          const float* src = p.part_o + (sl * hps + h) * D + d0;
          if constexpr (CPL == 4) {
            const float4 t4 = __ldcg(reinterpret_cast<const float4*>(src));
            v[k][0] = t4.x; v[k][1] = t4.y; v[k][2] = t4.z; v[k][3] = t4.w;
          } else {
            const float2 t2 = __ldcg(reinterpret_cast<const float2*>(src));
            v[k][0] = t2.x; v[k][1] = t2.y;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float mn = fmaxf(M[k], mlv[k].x);
          const float mu = (mn == -INFINITY) ? 0.f : mn;
          const float a = ptx::ex2(M[k] - mu), bw = ptx::ex2(mlv[k].x - mu);
          L[k] = L[k] * a + mlv[k].y * bw;
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[k][c] = acc[k][c] * a + v[k][c] * bw;
          M[k] = mn;
        }
      }
    };
    // Normalised bf16 row of out.
    auto store_row = [&](int b, int kvh, int row, float L, const float (&acc)[CPL]) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint16_t* dst = p.out + seq_row(b, kvh, row) * D + d0;
      if constexpr (CPL == 4) {
        uint2 u;
        u.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
        u.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = u;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
      }
    };
    // Arrival count of a segment's pieces (relaxed; a fence follows a count that shows
    // every other piece published, pairing with the publishers' fence before their add).
    auto arrivals = [&](int64_t segid) -> int { return lane == 0 ? ptx::ld_relaxed_gpu(p.counters + segid) : 0; };
    // The range's final piece, when cut, ends the CTA: if the segment's other pieces are
    // all published by then (they usually finished long before), their merged partial is
    // loaded while the consumers finish this one, and this CTA writes out without
    // publishing its own piece (no store, fence and arrival round trip, no reload).  The
    // count is read once on reaching the piece end and, if short, once more with the read
    // in flight during the wait for the consumers.
    bool pre = false;
    int late = 0;  // the second read
    // Merge the other pieces into the shared buffer (each lane its columns; the (max, sum)
    // pairs, equal in every lane, from lane 0).
    auto prefetch_others = [&](int64_t sbase, int64_t wf, int64_t wl, int nrows) {
      __threadfence();
      float M[8], L[8], acc[8][CPL];
      merge_pieces(sbase, wf, wl, w, 0, nrows, M, L, acc);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) pre_o[k * D + d0 + c] = acc[k][c];
        if (lane == 0) {
          pre_ml[2 * k] = M[k];
          pre_ml[2 * k + 1] = L[k];
        }
      }
      __syncwarp();
    };
    int64_t seg_base = x0 - cu.blk;  // linear index of block 0 of the current block's segment
    int e_blk0 = cu.blk;
    for (int64_t i = 0; i < total; ++i) {
      if (i == 0 || cu.blk == 0) e_blk0 = cu.blk;
      if ((cu.blk + 1 == cu.nblk) || (i + 1 == total)) {
        const int stage = static_cast<int>(i % S);
        // (the walk's block is the stage's: this piece's segment from the cursor)
        const bool final_cut = NT == 1 && (i + 1 == total) && !(e_blk0 == 0 && cu.blk + 1 == cu.nblk);
        if (final_cut) {
          const int64_t sb = seg_base;
          const int64_t wf = worker_of(sb, T, W), wl = worker_of(sb + cu.nblk - 1, T, W);
          const int64_t sid = static_cast<int64_t>(cu.b) * segs + cu.seg;
          if (__shfl_sync(0xffffffffu, arrivals(sid), 0) == static_cast<int>(wl - wf)) {
            pre = true;
            prefetch_others(sb, wf, wl, min(hps, grp - cu.ht * hps));
          } else {
            late = arrivals(sid);  // consumed after the wait
          }
        }
        const bool ok = ptx::mbar_wait_bounded(comb_bar + 8 * stage, (comb_phase >> stage) & 1u, limit);
        comb_phase ^= 1u << stage;
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) atomicOr(p.err, kErrTimeout);
          return;
        }
        const StageInfo si = info[stage];
        const float* ml = cml + stage * C * NH * 2;  // [C][NH][2]
        const uint8_t* st = base_ptr + stage * G_::kStageBytes;
        const int kvh = si.seg / p.n_ht, ht = si.seg % p.n_ht;
        const int nrows = min(hps, grp - ht * hps);
        const bool sole = si.flags & kSole;
        const float vscale = F8 ? __ldg(p.v_scales + kvh) : 1.f;
        const int64_t slot = w * 2 + ((si.flags & kFirstPieceOfCta) ? 0 : 1);
        // This piece's row h: the C consumers' states combined (max M, sum L, O acc).
        auto combine = [&](int h, float& M, float& L, float (&acc)[CPL]) {
          float mj[C], wj[C];
          M = -INFINITY;
          L = 0.f;
#pragma unroll
          for (int jj = 0; jj < C; ++jj) {
            mj[jj] = ml[(jj * NH + h) * 2];
            M = fmaxf(M, mj[jj]);
          }
#pragma unroll
          for (int jj = 0; jj < C; ++jj) {
            wj[jj] = (mj[jj] == -INFINITY) ? 0.f : ptx::ex2(mj[jj] - M);
            L += wj[jj] * ml[(jj * NH + h) * 2 + 1];
          }
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
#pragma unroll
          for (int jj = 0; jj < C; ++jj) {
            const float* src = reinterpret_cast<const float*>(st + jj * 2 * G_::kSubBytes +
                                                              (h >= HS ? G_::kSubBytes : 0)) + (h % HS) * D + d0;
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[c] += wj[jj] * src[c];
          }
          if constexpr (F8) {  // the cached V values are codes x the kv head's V scale
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[c] *= vscale;
          }
        };
        const int64_t segid = static_cast<int64_t>(si.b) * segs + si.seg;
        if (final_cut && !sole) {
          const int64_t wf = worker_of(si.seg_base, T, W), wl = worker_of(si.seg_base + si.nblk - 1, T, W);
          if (!pre && __shfl_sync(0xffffffffu, late, 0) == static_cast<int>(wl - wf)) {
            pre = true;
            prefetch_others(si.seg_base, wf, wl, nrows);
          }
          if (pre) {
            for (int h = 0; h < nrows; ++h) {
              float M, L, acc[CPL];
              combine(h, M, L, acc);
              const float pm = pre_ml[2 * h], pl = pre_ml[2 * h + 1];
              const float mn = fmaxf(M, pm);
              const float mu = (mn == -INFINITY) ? 0.f : mn;
              const float a = ptx::ex2(M - mu), bw = ptx::ex2(pm - mu);
              L = L * a + pl * bw;
#pragma unroll
              for (int c = 0; c < CPL; ++c) acc[c] = acc[c] * a + pre_o[h * D + d0 + c] * bw;
              store_row(si.b, kvh, ht * hps + h, L, acc);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              ptx::mbar_arrive_cnt(empty_bar + 8 * stage, C);
              p.counters[segid] = 0;  // every other piece has arrived: ready for the next launch
            }
            continue;  // the range's last block
          }
        }
        for (int h = 0; h < nrows; ++h) {
          float M, L, acc[CPL];
          combine(h, M, L, acc);
          if (sole) {
            store_row(si.b, kvh, ht * hps + h, L, acc);
          } else {
            float* dst = p.part_o + (slot * hps + h) * D + d0;
#pragma unroll
            for (int c = 0; c < CPL; ++c) dst[c] = acc[c];
            if (lane == 0)
              *reinterpret_cast<float2*>(p.part_ml + (slot * hps + h) * 2) = make_float2(M, L);
          }
        }
        // The stage is free again: all lanes are done reading it.
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cnt(empty_bar + 8 * stage, C);

        if (!sole) {
          // Cross-CTA step: the last CTA to finish its piece merges every piece.
          __threadfence();
          __syncwarp();
          int prev = 0;
          if (lane == 0) prev = atomicAdd(p.counters + segid, 1);
          prev = __shfl_sync(0xffffffffu, prev, 0);
          const int64_t wf = worker_of(si.seg_base, T, W);
          const int64_t wl = worker_of(si.seg_base + si.nblk - 1, T, W);
          if (prev == static_cast<int>(wl - wf)) {
            __threadfence();
            for (int h0 = 0; h0 < nrows; h0 += 8) {
              float M[8], L[8], acc[8][CPL];
              merge_pieces(si.seg_base, wf, wl, -1, h0, nrows, M, L, acc);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                if (h0 + k < nrows) store_row(si.b, kvh, ht * hps + h0 + k, L[k], acc[k]);
            }
            if (lane == 0) p.counters[segid] = 0;
          }
        }
      }
      if (i + 1 < total) {
        walk_next(cu, next_len, p, segs, cap);
        if (cu.blk == 0) seg_base = x0 + i + 1;
      }
    }
    return;
  }

  // ============================================================== consumer warps
  const int j = warp;
  // sub-chunk j's K tile within its K|V pair (V first when the paired map's lower pool is V)
  const uint32_t koff = p.kv_pair == 2 ? G_::kSubBytes : 0u;
  const int g = lane >> 2;
  const int q = lane & 3;
  uint32_t kofs[4], vofs[4];
  uint32_t ofs8[D / 32];   // F8: ldmatrix row addresses of K
  uint32_t vofs8[D / 32];  // F8: transposing byte ldmatrix row addresses of V
  if constexpr (F8) {
    // lane 16 m + j addresses token (j & 1) + 8 ((j >> 1) & 1) + 2 (j >> 2), 16-value chunk
    // 2 x + m, so that lane (g, q) receives tokens 2q, 2q+1, 2q+8, 2q+9
    {
      const int j = lane & 15;
      const int tok = (j & 1) + 8 * ((j >> 1) & 1) + 2 * (j >> 2);
#pragma unroll
      for (int x = 0; x < D / 32; ++x) {
        const int chunk = 2 * x + (lane >> 4);
        const int row = tok / (128 / D);
        const int c = (tok % (128 / D)) * (D / 16) + chunk;
        vofs8[x] = static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
      }
    }
    // lane l addresses row l % 8 of matrix l / 8: token (l % 8) + 8 ((l / 8) & 1), 16-value
    // chunk 2 x + (l / 16) of the x-th 32 values; a token's D codes are D / 128 of a
    // 128-byte swizzled row
    const int tok = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
    for (int x = 0; x < D / 32; ++x) {
      const int chunk = 2 * x + (lane >> 4);
      const int row = tok / (128 / D);
      const int c = (tok % (128 / D)) * (D / 16) + chunk;
      ofs8[x] = static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
    }
  }
  {
    // K as the A operand: matrices (t0-7, d), (t8-15, d), (t0-7, d+8), (t8-15, d+8).
    const int tokK = (lane & 7) + (((lane >> 3) & 1) << 3);
    const int yK = (lane >> 4) ^ (lane & 7);
    // V^T as the A operand: matrices (t0-7, d), (t0-7, d+8), (t8-15, d), (t8-15, d+8).
    const int tokV = (lane & 7) + ((lane >> 4) << 3);
    const int yV = ((lane >> 3) & 1) ^ (lane & 7);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      kofs[jj] = static_cast<uint32_t>(tokK * 128 + (((2 * jj) ^ yK) << 4));
      vofs[jj] = static_cast<uint32_t>(tokV * 128 + (((2 * jj) ^ yV) << 4));
    }
  }

  uint32_t qf[MT][NT][2];
  float o[MT][NT][4];
  float mref[NT][2], lsum[NT][2];
  int nrows_seg = 0;  // valid heads of the segment
  int nrows_c = 0;    // valid heads of this consumer's tile
  int cdrop[NT][2];   // MQ: query tokens newer than each column's own
  const int max_drop = MQ ? p.q_len - 1 : 0;
  float sl2 = p.scale_log2;

  auto load_q = [&](int b, int seg, int stage) {
    const int kvh = seg / p.n_ht;
    const int ht = seg % p.n_ht;
    if constexpr (F8) sl2 = p.scale_log2 * __ldg(p.k_scales + kvh);
    nrows_seg = min(p.heads_per_seg, grp - ht * p.heads_per_seg);
    nrows_c = min(NH, nrows_seg);
    const int r0 = ht * p.heads_per_seg;  // first row of the segment
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        cdrop[nt][e] = MQ ? max_drop - (r0 + nt * 8 + 2 * q + e) / p.group : 0;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
      const bool v = h < nrows_c;
      // from the rows staged with the piece's first block
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qbuf + stage * kQBytes) + (v ? h : 0) * (D / 2);
#pragma unroll
      for (int ks = 0; ks < MT; ++ks) {
        if constexpr (F8) {  // fp16, values 16 ks + 4q, +1 and 16 ks + 4q + 2, +3 (the K order)
          qf[ks][nt][0] = v ? ptx::bf16x2_to_f16x2(qrow[ks * 8 + 2 * q]) : 0u;
          qf[ks][nt][1] = v ? ptx::bf16x2_to_f16x2(qrow[ks * 8 + 2 * q + 1]) : 0u;
        } else {
          qf[ks][nt][0] = v ? qrow[ks * 8 + q] : 0u;
          qf[ks][nt][1] = v ? qrow[ks * 8 + 4 + q] : 0u;
        }
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mref[nt][0] = mref[nt][1] = -INFINITY;
      lsum[nt][0] = lsum[nt][1] = 0.f;
    }
  };


  for (int64_t i = 0; i < total; ++i) {
    const int stage = static_cast<int>(i % S);
    const bool arrived = ptx::mbar_wait_bounded(full_bar + 8 * stage, static_cast<uint32_t>((i / S) & 1), limit);
    if (!__all_sync(0xffffffffu, arrived)) {
      if (lane == 0) atomicOr(p.err, kErrTimeout);
      return;
    }
    const StageInfo si = info[stage];
    if (si.flags & kFirstOfPiece) load_q(si.b, si.seg, stage);

    if ((si.submask >> j) & 1) {
      const uint32_t sub = ring + stage * G_::kStageBytes + j * 2 * G_::kSubBytes;
      const uint32_t kb = sub + koff, vb = sub + (G_::kSubBytes - koff);
      if constexpr (F8)
        attend_subchunk_f8<D, NT>(kb, vb, min(kChunk, si.nvalid - j * kChunk), ofs8, vofs8, qf, o, mref,
                                  lsum, sl2, g, q);
      else
        attend_subchunk<D, NT, MQ>(kb, vb, min(kChunk, si.nvalid - j * kChunk),
                                   kofs, vofs, qf, o, mref, lsum, sl2, g, q, si.rem - j * kChunk, max_drop,
                                   cdrop);
    }
    const bool piece_end = si.flags & kLastOfPiece;
    __syncwarp();
    // A piece end keeps the stage: the epilogue warp releases it after the combine (it
    // arrives for all C consumers).
    if (lane == 0 && !piece_end) ptx::mbar_arrive(empty_bar + 8 * stage);

    if (!piece_end) continue;

    // ------------------------------------------------------------ end of a piece
    float lt[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lsum[nt][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        lt[nt][e] = l;
      }
    const bool sole = si.flags & kSole;
    const int hps = p.heads_per_seg;
    const int kvh = si.seg / p.n_ht;
    const int ht = si.seg % p.n_ht;
    const int slot = static_cast<int>(w * 2 + ((si.flags & kFirstPieceOfCta) ? 0 : 1));

    {
      // Hand the piece to the epilogue warp.  This consumer's partial O^T
      // (relative to its own reference max) goes into the tiles of its sub-chunk, which
      // only it read; its (max, sum) pairs into cml[stage][j].
      float* mlj = cml + (stage * C + j) * NH * 2;
      if (g == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = nt * 8 + 2 * q + e;
            mlj[h * 2] = mref[nt][e];
            mlj[h * 2 + 1] = lt[nt][e];
          }
      }
      // Head h of this consumer goes to the first tile of its sub-chunk (h < HS) or the
      // second.  O^T M-row g of tile mt is dimension 16 mt + g (row g + 8: 16 mt + g + 8).
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = nt * 8 + 2 * q + e;
          float* row = reinterpret_cast<float*>(base_ptr + stage * G_::kStageBytes + j * 2 * G_::kSubBytes +
                                                (h >= HS ? G_::kSubBytes : 0)) + (h % HS) * D;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            row[mt * 16 + g] = o[mt][nt][e];
            row[mt * 16 + g + 8] = o[mt][nt][e + 2];
          }
        }
      }
      ptx::fence_proxy_async_smem();  // the stage will be refilled by TMA later
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(comb_bar + 8 * stage);
    }
  }
}

// ------------------------------------------------------------------ host side
namespace {


template <int D, int NT, int C, bool F8 = false>
struct Cfg {
  static constexpr int kNH = 8 * NT;
  // per stage: K/V tiles, the piece's query rows, the consumers' (max, sum) hand-off
  static constexpr size_t kQBytes = static_cast<size_t>(kNH) * D * 2;
  static constexpr size_t kMergePerStage = static_cast<size_t>(C * kNH * 2) * sizeof(float);
  static constexpr size_t kBudget = F8 ? static_cast<size_t>(GQA_F8_SMEM_PER_SM_KB) * 1024 / kWsCtasPerSmF8
                                      : static_cast<size_t>(GQA_SMEM_PER_SM_KB) * 1024 / kWsCtasPerSm;
  static constexpr int kStagesRaw =
      static_cast<int>(kBudget / (Geo<D, F8>::kStageBytes + kQBytes + kMergePerStage));
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr size_t kMerge = kStages * kMergePerStage;
  // one n-tile: the epilogue's merged partial of the other pieces of its final segment
  // ([8][D] O and 8 (max, sum) pairs, 16-byte aligned), outside the stage budget
  static constexpr size_t kPre = NT == 1 ? (8 * D + 16) * sizeof(float) + 16 : 0;
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * (Geo<D, F8>::kStageBytes + kQBytes) +
                                  kMerge + kStages * (sizeof(StageInfo) + 24) + kPre;
};

template <int D, int NT, int C, bool MQ, bool F8 = false>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                     cudaStream_t stream, bool overlap) {
  using CF = Cfg<D, NT, C, F8>;
  auto kern = decode_ws_kernel<D, NT, C, CF::kStages, MQ, F8>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(CF::kSmem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const int threads = (C + 2) * 32;  // consumers, producer, epilogue
  if (!overlap) {
    kern<<<grid, threads, CF::kSmem, stream>>>(tk, tv, p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = CF::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, p);
}

template <int D, bool MQ>
cudaError_t launch_d(const DecodeParams& p, const DecodePlan& pl, const CUtensorMap& tk,
                     const CUtensorMap& tv, int grid, cudaStream_t s, bool o) {
  return pl.n_tiles == 1 ? launch_t<D, 1, 4, MQ>(p, tk, tv, grid, s, o) : launch_t<D, 2, 4, MQ>(p, tk, tv, grid, s, o);
}

template <int D, int NT, int C, bool F8 = false>
void fill(DecodePlan& pl) {
  using CF = Cfg<D, NT, C, F8>;
  pl.stages = CF::kStages;
  pl.smem_bytes = CF::kSmem;
}

}  // namespace

// Small groups (G <= 16): token split, 4 consumers, one 8- or 16-head tile per segment.
// Larger groups run on the tcgen05 kernel (decode_tc.cu), one 128-row MMA tile of heads
// per segment: from 17 heads on its per-block cost (fixed by the 128-row tile) is below
// the mma.sync kernel's, whose work grows with the heads (measured: 24 and 32 heads per
// kv head, 29-49 us against 46-73 us).  Rows of several query tokens per sequence
// (mq_rows) follow the same rule; on the tcgen05 kernel they form one segment (<= 128).
DecodePlan plan_decode(int head_dim, int group, bool mq_rows, bool fp8) {
  DecodePlan pl{};
  (void)mq_rows;
  if (fp8 && group <= 16) {
    // 8-bit cache: a consumer's 8-head partial fills both its K and V sub-chunk tiles, so
    // a segment is one 8-head tile; 9 to 16 heads per kv head take two segments (each
    // reads the kv head's codes).
    pl.n_tiles = 1;
    pl.consumers = 4;
    pl.heads_per_seg = 8;
    pl.n_ht = (group + 7) / 8;
    pl.ctas_per_sm = kWsCtasPerSmF8;
    if (head_dim == 64) fill<64, 1, 4, true>(pl); else fill<128, 1, 4, true>(pl);
    return pl;
  }
  if (group > 16) {
    // Dense enough for the 5th-generation tensor cores: one 128-row MMA tile of heads.
    pl.tensor_cores = 1;
    pl.heads_per_seg = group < 128 ? group : 128;
    pl.n_ht = (group + pl.heads_per_seg - 1) / pl.heads_per_seg;
    pl.ctas_per_sm = 1;
    pl.consumers = 4;
    pl.smem_bytes = decode_tc_smem_bytes(head_dim, fp8);
    return pl;
  }
  pl.n_tiles = group <= 8 ? 1 : 2;
  pl.consumers = 4;
  pl.heads_per_seg = 8 * pl.n_tiles;
  pl.n_ht = 1;
  pl.ctas_per_sm = kWsCtasPerSm;
  if (head_dim == 64) {
    if (pl.n_tiles == 1) fill<64, 1, 4>(pl); else fill<64, 2, 4>(pl);
  } else {
    if (pl.n_tiles == 1) fill<128, 1, 4>(pl); else fill<128, 2, 4>(pl);
  }
  return pl;
}

cudaError_t launch_decode(const DecodeParams& p, const DecodePlan& pl, const CUtensorMap& tk,
                          const CUtensorMap& tv, int grid, cudaStream_t stream, bool overlap) {
  if (p.k_scales != nullptr)
    return p.head_dim == 64 ? launch_t<64, 1, 4, false, true>(p, tk, tv, grid, stream, overlap)
                            : launch_t<128, 1, 4, false, true>(p, tk, tv, grid, stream, overlap);
  if (p.q_len > 1)
    return p.head_dim == 64 ? launch_d<64, true>(p, pl, tk, tv, grid, stream, overlap)
                            : launch_d<128, true>(p, pl, tk, tv, grid, stream, overlap);
  if (p.head_dim == 64) return launch_d<64, false>(p, pl, tk, tv, grid, stream, overlap);
  return launch_d<128, false>(p, pl, tk, tv, grid, stream, overlap);
}

}  // namespace gqa
