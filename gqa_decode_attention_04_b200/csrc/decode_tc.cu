// Paged decode attention for large query groups (MQA-like: many query heads per K/V head)
// on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// Same result as decode_ws.cu (page "TensorRT对Multi-Query Attention的专项优化支持": decode
// re-reads all cached K/V; with MQA every query head shares one K/V head, which the plugin
// computes "without unnecessary copying and broadcasting" of K/V, on tensor cores for QK^T
// and AV with tiled shared-memory prefetch; tiny-llm "优化" page: paged KV by block table,
// FlashDecoding for long contexts).  With G query heads per K/V head the contraction is
// G flop per cached byte; for G = 96 this is a dense GEMM that CUDA-core or mma.sync code
// cannot keep up with at HBM speed, so it runs on tcgen05:
//
//   * Work list and split: as decode_ws.cu, with 64-token blocks; one contiguous range of
//     the (sequence, segment, block) list per CTA, one CTA per SM; a segment covers up to
//     128 query heads (the MMA's M = 128 rows), more heads use more segments.
//   * Producer warp: TMA copies of each block's K and V ([64 tokens, 64 dims] boxes,
//     128-byte swizzle, K-major for K, MN-major use for V) into a ring of stages, and of
//     the segment's 128 query rows into a double-buffered Q tile at each piece start.
//   * MMA warp (one thread issues): S_j = Q K_j^T (M=128 heads, N=64 tokens, K=head_dim)
//     into one of two TMEM buffers; then O += P_{j-1} V_{j-1} with P read from TMEM
//     (M=128, N=head_dim, K=64 tokens).  Completion is signalled with tcgen05.commit.
//   * Softmax warpgroup (128 threads, thread r = query head r): reads its S row from TMEM,
//     online softmax in the log2 domain with a lazily moved reference (O rescaled in TMEM
//     only when the row maximum rises by more than 8), writes P (bf16) over S in TMEM.
//     At a piece end it reads its O row, normalises it and writes out, or stores the
//     piece for the cross-CTA log-sum-exp merge (last CTA to finish merges).
//   * Safety: every wait is bounded; on a timeout all warps leave their loops, the MMA
//     warp waits for its issued MMAs, and TMEM is released before exit.
#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kTcBlk = 64;      // tokens per stage
constexpr int kTcRows = 128;    // MMA M: query-head rows per segment
constexpr uint32_t kTmemCols = 256;
constexpr float kTcRescale = 8.0f;

template <int D>
struct TcGeo {
  static constexpr int kGroups = D / 64;                 // 64-column (128-byte) groups
  static constexpr int kGroupBytes = kTcBlk * 128;       // 64 rows x 128 bytes
  static constexpr int kTile = kGroups * kGroupBytes;    // K (or V) of one block
  static constexpr int kStage = 2 * kTile;
  static constexpr int kQGroup = kTcRows * 128;
  static constexpr int kQTile = kGroups * kQGroup;
  static constexpr int kStages = D == 128 ? 4 : 8;
  // TMEM columns: S/P buffers 0 and 1 at 0 and 64 (64 fp32 columns each; P, bf16 pairs,
  // overwrites the first 32), O at 128 (D columns).
  static constexpr uint32_t kS0 = 0, kS1 = 64, kO = 128;
};

struct TcStageInfo {
  int64_t seg_base;
  uint64_t vmask;  // bit t: token t of the block is inside the sequence and its page was loaded
  int b, seg, blk, nblk, nvalid, flags, piece, pad;
};
enum : int { kTcFirst = 1, kTcLast = 2, kTcSole = 4, kTcFirstPieceOfCta = 8 };

__device__ __forceinline__ int tc_eff_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }
__device__ __forceinline__ int64_t tc_wstart(int64_t w, int64_t T, int64_t W) { return w * T / W; }
__device__ __forceinline__ int64_t tc_worker_of(int64_t x, int64_t T, int64_t W) { return ((x + 1) * W - 1) / T; }

struct TcCursor {
  int b, seg, blk, nblk, len;
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(192, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                 const __grid_constant__ CUtensorMap tmap_q, const DecodeParams p) {
  using GE = TcGeo<D>;
  constexpr int S = GE::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_wtot[6];
  __shared__ int s_start_b;
  __shared__ int64_t s_start_base;
  __shared__ uint32_t s_tmem;
  __shared__ int s_prev;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.num_seqs;
  const int segs = p.num_kv_heads * p.n_ht;
  const int cap = p.max_blocks * p.page_size;
  const int hps = p.heads_per_seg;

  // ---------------------------------------------------------------- prologue (split)
  int64_t mine = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = __ldg(p.seq_lens + b);
    const int Le = tc_eff_len(L, cap);
    if ((L < 0 || L > cap) && blockIdx.x == 0) atomicOr(p.err, kErrBounds);
    if (Le == 0 && (b % gridDim.x) == blockIdx.x) {
      uint32_t* o = reinterpret_cast<uint32_t*>(p.out + static_cast<int64_t>(b) * p.num_heads * D);
      for (int i = 0; i < p.num_heads * D / 2; ++i) o[i] = 0u;
    }
    mine += static_cast<int64_t>((Le + kTcBlk - 1) / kTcBlk) * segs;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if (lane == 0) s_wtot[warp] = mine;
  if (threadIdx.x == 0) {
    s_start_b = -1;
    s_abort = 0;
  }
  __syncthreads();
  int64_t T = 0;
  for (int i = 0; i < 6; ++i) T += s_wtot[i];
  const int64_t W = min(static_cast<int64_t>(p.num_workers), T);
  const int64_t w = blockIdx.x;
  if (w >= W) return;
  const int64_t x0 = tc_wstart(w, T, W), x1 = tc_wstart(w + 1, T, W);
  __syncthreads();
  {
    int64_t base = 0;
    for (int t0 = 0; t0 < B && base <= x0; t0 += blockDim.x) {
      const int b = t0 + threadIdx.x;
      int64_t n = 0;
      if (b < B) n = static_cast<int64_t>((tc_eff_len(__ldg(p.seq_lens + b), cap) + kTcBlk - 1) / kTcBlk) * segs;
      int64_t incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (lane == 31) s_wtot[warp] = incl;
      __syncthreads();
      int64_t pre = 0, tot = 0;
      for (int i = 0; i < 6; ++i) {
        if (i < warp) pre += s_wtot[i];
        tot += s_wtot[i];
      }
      incl += pre;
      if (n > 0 && x0 >= base + incl - n && x0 < base + incl) {
        s_start_b = b;
        s_start_base = base + incl - n;
      }
      base += tot;
      __syncthreads();
    }
  }
  if (s_start_b < 0) {  // cannot happen for a non-empty range
    if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
    return;
  }

  // ---------------------------------------------------------------- shared layout
  const uint32_t smem0 = ptx::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (smem0 & 1023u)) & 1023u;
  uint8_t* base_ptr = smem_raw + pad;
  const uint32_t ring = smem0 + pad;                        // S stages of K | V
  const uint32_t qbuf = ring + S * GE::kStage;              // 2 Q tiles
  uint8_t* vring = base_ptr;                                // generic view of the ring
  TcStageInfo* info = reinterpret_cast<TcStageInfo*>(base_ptr + S * GE::kStage + 2 * GE::kQTile);
  const uint32_t bar0 = ptx::smem_u32(info + S);
  const uint32_t full_bar = bar0;                 // [S] producer -> MMA (K/V landed)
  const uint32_t empty_bar = full_bar + 8 * S;    // [S] MMA commit -> producer
  const uint32_t qfull_bar = empty_bar + 8 * S;   // [2]
  const uint32_t qempty_bar = qfull_bar + 16;     // [2]
  const uint32_t sfull_bar = qempty_bar + 16;     // [2] MMA commit -> softmax
  const uint32_t pfull_bar = sfull_bar + 16;      // [2] softmax (128) -> MMA
  const uint32_t pv_bar = pfull_bar + 16;         // MMA commit after each PV
  const uint32_t ofree_bar = pv_bar + 8;          // softmax (128) -> MMA, after a piece's O is read
  const uint32_t drain_bar = ofree_bar + 8;       // MMA commit at exit
  const uint32_t wg_bar = drain_bar + 8;          // softmax warpgroup rendezvous (128)

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar + 8 * s, 1);
      ptx::mbar_init(empty_bar + 8 * s, 1);
    }
    for (int k = 0; k < 2; ++k) {
      ptx::mbar_init(qfull_bar + 8 * k, 1);
      ptx::mbar_init(qempty_bar + 8 * k, 1);
      ptx::mbar_init(sfull_bar + 8 * k, 1);
      ptx::mbar_init(pfull_bar + 8 * k, 128);
    }
    ptx::mbar_init(pv_bar, 1);
    ptx::mbar_init(ofree_bar, 128);
    ptx::mbar_init(drain_bar, 1);
    ptx::mbar_init(wg_bar, 128);
    ptx::fence_mbarrier_init();
  }
  if (warp == 5) ptx::tmem_alloc(ptx::smem_u32(&s_tmem), kTmemCols);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s_tmem;

  const int64_t total = x1 - x0;
  const uint64_t limit = p.wait_limit_ns;
  TcCursor cu;
  cu.b = s_start_b;
  cu.len = tc_eff_len(__ldg(p.seq_lens + cu.b), cap);
  cu.nblk = (cu.len + kTcBlk - 1) / kTcBlk;
  {
    const int64_t off = x0 - s_start_base;
    cu.seg = static_cast<int>(off / cu.nblk);
    cu.blk = static_cast<int>(off % cu.nblk);
  }
  auto aborted = [&]() -> bool { return *reinterpret_cast<volatile int*>(&s_abort) != 0; };
  auto abort_all = [&](uint32_t bit) {
    atomicOr(p.err, bit);
    atomicExch(&s_abort, 1);
  };

  if (warp == 4) {
    // ============================================================ producer warp
    const uint64_t policy = ptx::policy_evict_first();
    const int ps = p.page_size;
    const int R = ps < kTcBlk ? ps : kTcBlk;   // rows per TMA box (one page or one block)
    const int nchunks = kTcBlk / R;           // lanes < nchunks each copy one box row range
    int next_len = (cu.b + 1 < B) ? __ldg(p.seq_lens + cu.b + 1) : 0;
    int64_t seg_base = x0 - cu.blk;
    int piece = 0;
    bool first_piece = true;
    int piece_blk0 = cu.blk;
    int64_t i = 0;
    for (; i < total; ++i) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      const int stage = static_cast<int>(i % S);
      if (i >= S) {
        const bool ok = ptx::mbar_wait_bounded(empty_bar + 8 * stage, static_cast<uint32_t>((i / S - 1) & 1), limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
      }
      const bool first = (i == 0) || cu.blk == 0;
      const bool last = (i + 1 == total) || (cu.blk + 1 == cu.nblk);
      if (first) piece_blk0 = cu.blk;
      const int kvh = cu.seg / p.n_ht, ht = cu.seg % p.n_ht;
      if (first) {
        // Q rows of this piece's segment into buffer piece & 1 (freed by the MMA warp).
        const int qb = piece & 1;
        bool ok = true;
        if (piece >= 2)
          ok = ptx::mbar_wait_bounded(qempty_bar + 8 * qb, static_cast<uint32_t>((piece / 2 - 1) & 1), limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
        if (lane == 0) {
          if (i == 0) ptx::pdl_wait_prerequisites();
          ptx::mbar_arrive_expect_tx(qfull_bar + 8 * qb, p.arm_without_copy ? 1u : GE::kQTile);
          if (!p.arm_without_copy) {
            const int row0 = cu.b * p.num_heads + kvh * p.group + ht * hps;
#pragma unroll
            for (int g = 0; g < GE::kGroups; ++g)
              ptx::tma_load_3d(qbuf + qb * GE::kQTile + g * GE::kQGroup, &tmap_q, qfull_bar + 8 * qb, 0, row0, g, 0);
          }
        }
      }
      const int nvalid = min(kTcBlk, cu.len - cu.blk * kTcBlk);
      int page = -1;
      const bool want = lane < nchunks && lane * R < nvalid;
      if (want) {
        const int t = cu.blk * kTcBlk + lane * R;
        page = __ldg(p.block_table + static_cast<int64_t>(cu.b) * p.max_blocks + t / ps);
      }
      const bool ok = want && page >= 0 && page < p.num_pages;
      if (__any_sync(0xffffffffu, want && !ok) && lane == 0) atomicOr(p.err, kErrBounds);
      const uint32_t okbits = __ballot_sync(0xffffffffu, ok);
      const uint32_t nload = __popc(okbits);
      uint64_t vmask = 0;
      for (int c = 0; c < nchunks; ++c)
        if ((okbits >> c) & 1u) vmask |= (R >= 64 ? ~0ull : ((1ull << R) - 1ull)) << (c * R);
      if (nvalid < kTcBlk) vmask &= (1ull << nvalid) - 1ull;
      if (lane == 0) {
        TcStageInfo& si = info[stage];
        si.seg_base = seg_base;
        si.vmask = vmask;
        si.b = cu.b;
        si.seg = cu.seg;
        si.blk = cu.blk;
        si.nblk = cu.nblk;
        si.nvalid = nvalid;
        si.piece = piece;
        si.flags = (first ? kTcFirst : 0) | (last ? kTcLast : 0) |
                   ((last && piece_blk0 == 0 && cu.blk + 1 == cu.nblk) ? kTcSole : 0) |
                   (first_piece ? kTcFirstPieceOfCta : 0);
        const uint32_t bytes = p.arm_without_copy ? 0u : nload * 2u * GE::kGroups * R * 128u;
        if (bytes) ptx::mbar_arrive_expect_tx(full_bar + 8 * stage, bytes);
        else if (p.arm_without_copy) ptx::mbar_arrive_expect_tx(full_bar + 8 * stage, 1u);
        else ptx::mbar_arrive(full_bar + 8 * stage);
      }
      if (i == 0 && lane == 0 && !first) ptx::pdl_wait_prerequisites();
      __syncwarp();
      if (ok && !p.arm_without_copy) {
        const int t = cu.blk * kTcBlk + lane * R;
        const int row = (page * p.num_kv_heads + kvh) * ps + t % ps;
        const uint32_t kdst = ring + stage * GE::kStage + lane * R * 128;
        const uint32_t vdst = kdst + GE::kTile;
#pragma unroll
        for (int g = 0; g < GE::kGroups; ++g) {
          ptx::tma_load_3d(kdst + g * GE::kGroupBytes, &tmap_k, full_bar + 8 * stage, 0, row, g, policy);
          ptx::tma_load_3d(vdst + g * GE::kGroupBytes, &tmap_v, full_bar + 8 * stage, 0, row, g, policy);
        }
      }
      if (last) {
        first_piece = false;
        ++piece;
      }
      if (i + 1 < total) {
        if (++cu.blk >= cu.nblk) {
          cu.blk = 0;
          if (++cu.seg >= segs) {
            cu.seg = 0;
            do {
              ++cu.b;
              cu.len = (cu.b < B) ? tc_eff_len(next_len, cap) : 0;
              cu.nblk = (cu.len + kTcBlk - 1) / kTcBlk;
              next_len = (cu.b + 1 < B) ? __ldg(p.seq_lens + cu.b + 1) : 0;
            } while (cu.nblk == 0 && cu.b + 1 < B);
          }
          seg_base = x0 + i + 1;
        }
      }
    }
    // Let copies still in flight land before the CTA can exit.
    for (int64_t j = (i > S ? i - S : 0); j < i; ++j)
      ptx::mbar_wait_bounded(full_bar + 8 * (j % S), static_cast<uint32_t>((j / S) & 1), limit);
  } else if (warp == 5) {
    // ============================================================ MMA warp
    constexpr uint32_t idS = ptx::umma_idesc_bf16(kTcRows, kTcBlk, false);
    constexpr uint32_t idPV = ptx::umma_idesc_bf16(kTcRows, D, true);
    int64_t pend = -1;            // block whose P V is not issued yet
    int pend_stage = 0, pend_first = 0, pend_piece = 0;
    uint64_t pend_vmask = 0;
    bool failed = false;
    // O += P_j V_j for a pending block j.
    auto issue_pv = [&](int64_t j, int stage, uint64_t vmask, int first, int piece) -> bool {
      const int sb = static_cast<int>(j & 1);
      bool ok = ptx::mbar_wait_bounded(pfull_bar + 8 * sb, static_cast<uint32_t>((j / 2) & 1), limit);
      if (ok && first && piece > 0)  // the previous piece's O has been read out
        ok = ptx::mbar_wait_bounded(ofree_bar, static_cast<uint32_t>((piece - 1) & 1), limit);
      if (!__all_sync(0xffffffffu, ok)) return false;
      if (vmask != ~0ull) {
        // Rows of tokens past the sequence end (or of pages that failed the range check)
        // may hold any bits, NaN included: zero them in V so 0 * NaN cannot reach O.
        // (Their scores are masked to -inf by the softmax.)
        uint8_t* v = vring + stage * GE::kStage + GE::kTile;
        for (int idx = lane; idx < kTcBlk * 8 * GE::kGroups; idx += 32) {
          const int g = idx / (kTcBlk * 8);
          const int r = (idx / 8) % kTcBlk, c = idx % 8;
          if (!((vmask >> r) & 1ull))
            *reinterpret_cast<uint4*>(v + g * GE::kGroupBytes + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
      }
      ptx::tc_fence_after();
      if (lane == 0) {
        const uint32_t vb = ring + stage * GE::kStage + GE::kTile;
        const uint32_t pt = tmem + (sb ? GE::kS1 : GE::kS0);
#pragma unroll
        for (int ks = 0; ks < kTcBlk / 16; ++ks) {
          const uint64_t bdesc = ptx::umma_desc_sw128(vb + ks * 16 * 128, GE::kGroupBytes, 1024);
          ptx::umma_ts(tmem + GE::kO, pt + ks * 8, bdesc, idPV, (first && ks == 0) ? 0u : 1u);
        }
        ptx::umma_commit(empty_bar + 8 * stage);  // K_j and V_j are consumed
        ptx::umma_commit(pv_bar);
      }
      __syncwarp();
      return true;
    };
    for (int64_t i = 0; i < total && !failed; ++i) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      const int stage = static_cast<int>(i % S);
      bool ok = ptx::mbar_wait_bounded(full_bar + 8 * stage, static_cast<uint32_t>((i / S) & 1), limit);
      const TcStageInfo si = info[stage];
      const int qb = si.piece & 1;
      if (ok && (si.flags & kTcFirst))
        ok = ptx::mbar_wait_bounded(qfull_bar + 8 * qb, static_cast<uint32_t>((si.piece / 2) & 1), limit);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) abort_all(kErrTimeout);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const int sb = static_cast<int>(i & 1);
      if (lane == 0) {
        const uint32_t kb = ring + stage * GE::kStage;
        const uint32_t qt = qbuf + qb * GE::kQTile;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t a = ptx::umma_desc_sw128(qt + (ks >> 2) * GE::kQGroup + (ks & 3) * 32, 16, 1024);
          const uint64_t b = ptx::umma_desc_sw128(kb + (ks >> 2) * GE::kGroupBytes + (ks & 3) * 32, 16, 1024);
          ptx::umma_ss(tmem + (sb ? GE::kS1 : GE::kS0), a, b, idS, ks > 0 ? 1u : 0u);
        }
        ptx::umma_commit(sfull_bar + 8 * sb);
        if (si.flags & kTcLast) ptx::umma_commit(qempty_bar + 8 * qb);  // Q tile no longer read
      }
      __syncwarp();
      if (pend >= 0) {
        if (!issue_pv(pend, pend_stage, pend_vmask, pend_first, pend_piece)) {
          if (lane == 0) abort_all(kErrTimeout);
          failed = true;
          break;
        }
        pend = -1;
      }
      pend = i;
      pend_stage = stage;
      pend_vmask = si.vmask;
      pend_first = (si.flags & kTcFirst) ? 1 : 0;
      pend_piece = si.piece;
      if (si.flags & kTcLast) {  // finish the piece now so its O can be read out
        if (!issue_pv(pend, pend_stage, pend_vmask, pend_first, pend_piece)) {
          if (lane == 0) abort_all(kErrTimeout);
          failed = true;
          break;
        }
        pend = -1;
      }
    }
    // Every MMA issued by this warp completes before TMEM can be released.
    if (lane == 0) ptx::umma_commit(drain_bar);
    __syncwarp();
    ptx::mbar_wait_bounded(drain_bar, 0, limit);
  } else {
    // ============================================================ softmax warpgroup
    const int r = threadIdx.x;              // query-head row of the segment tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    const float sl2 = p.scale_log2;
    float mref = -INFINITY, lsum = 0.f;
    int64_t pv_seen = 0;  // PV completions consumed (one per block, in order)
    int wg_phase = 0;
    bool failed = false;
    // Every wait outcome is made warp-uniform: the TMEM loads and stores that follow are
    // warp-collective (.sync.aligned) and must never run on part of a warp.
    auto wait_pv_upto = [&](int64_t n) -> bool {
      while (pv_seen < n) {
        const bool ok = ptx::mbar_wait_bounded(pv_bar, static_cast<uint32_t>(pv_seen & 1), limit);
        if (!__all_sync(0xffffffffu, ok)) return false;
        ++pv_seen;
      }
      return true;
    };
    auto wg_sync = [&]() -> bool {  // all 128 threads (bounded)
      ptx::mbar_arrive(wg_bar);
      const bool ok = ptx::mbar_wait_bounded(wg_bar, static_cast<uint32_t>(wg_phase & 1), limit);
      ++wg_phase;
      return __all_sync(0xffffffffu, ok);
    };
    for (int64_t i = 0; i < total && !failed; ++i) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      const int sb = static_cast<int>(i & 1);
      bool ok = __all_sync(0xffffffffu,
                           ptx::mbar_wait_bounded(sfull_bar + 8 * sb, static_cast<uint32_t>((i / 2) & 1), limit));
      if (ok && i > 0) ok = wait_pv_upto(i);  // P_{i-1} V_{i-1} is in O
      if (!ok) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const TcStageInfo si = info[i % S];
      const bool first = si.flags & kTcFirst;
      if (first) {
        mref = -INFINITY;
        lsum = 0.f;
      }
      const uint32_t st = tmem + lane_off + (sb ? GE::kS1 : GE::kS0);
      uint32_t u0[32], u1[32];
      ptx::tmem_ld32(st, u0);
      ptx::tmem_ld32(st + 32, u1);
      ptx::tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = ((si.vmask >> c) & 1ull) ? __uint_as_float(u0[c]) * sl2 : -INFINITY;
        s[32 + c] = ((si.vmask >> (32 + c)) & 1ull) ? __uint_as_float(u1[c]) * sl2 : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) mx = fmaxf(mx, s[c]);
      const bool need = mx > mref + kTcRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ptx::ex2(mref - mx) : 1.f;  // 0 when mref = -inf
        if (!first) {
          // Rescale O rows in TMEM (P V of earlier blocks are complete).  The whole warp
          // takes part; rows that keep their reference scale by 1.
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            ptx::tmem_ld32(tmem + lane_off + GE::kO + c0, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            ptx::tmem_st32(tmem + lane_off + GE::kO + c0, ov);
          }
          ptx::tmem_wait_st();
        }
        if (need) {
          lsum *= alpha;
          mref = mx;
        }
      }
      const float mu = (mref == -INFINITY) ? 0.f : mref;
      uint32_t pk[32];
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float a = ptx::ex2(s[2 * c] - mu), b2 = ptx::ex2(s[2 * c + 1] - mu);
        ls += a + b2;
        pk[c] = ptx::pack_bf16x2(a, b2);
      }
      lsum += ls;
      ptx::tmem_st32(st, pk);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(pfull_bar + 8 * sb);

      if (!(si.flags & kTcLast)) continue;
      // ---------------------------------------------------------- end of a piece
      if (!wait_pv_upto(i + 1)) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const int kvh = si.seg / p.n_ht, ht = si.seg % p.n_ht;
      const int nrows = min(hps, p.group - ht * hps);
      const int64_t row0 = static_cast<int64_t>(si.b) * p.num_heads + kvh * p.group + ht * hps;
      const bool sole = si.flags & kTcSole;
      const int64_t slot = w * 2 + ((si.flags & kTcFirstPieceOfCta) ? 0 : 1);
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        ptx::tmem_ld32(tmem + lane_off + GE::kO + c0, ov);
        ptx::tmem_wait_ld();
        if (r < nrows) {
          if (sole) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (row0 + r) * D + c0);
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = ptx::pack_bf16x2(__uint_as_float(ov[c]) * inv, __uint_as_float(ov[c + 1]) * inv);
              v.y = ptx::pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
              v.z = ptx::pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
              v.w = ptx::pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
              dst[c / 8] = v;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(p.part_o + (slot * hps + r) * D + c0);
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              dst[c / 4] = make_float4(__uint_as_float(ov[c]), __uint_as_float(ov[c + 1]),
                                       __uint_as_float(ov[c + 2]), __uint_as_float(ov[c + 3]));
          }
        }
      }
      if (!sole && r < nrows)
        *reinterpret_cast<float2*>(p.part_ml + (slot * hps + r) * 2) = make_float2(mref, lsum);
      ptx::tc_fence_before();
      ptx::mbar_arrive(ofree_bar);  // O may be overwritten by the next piece
      if (sole) continue;
      // Cross-CTA step: the last CTA to finish its piece of the segment merges them all.
      __threadfence();
      if (!wg_sync()) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      const int64_t segid = static_cast<int64_t>(si.b) * segs + si.seg;
      if (r == 0) s_prev = atomicAdd(p.counters + segid, 1);
      if (!wg_sync()) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      const int prev = s_prev;
      const int64_t wf = tc_worker_of(si.seg_base, T, W);
      const int64_t wl = tc_worker_of(si.seg_base + si.nblk - 1, T, W);
      if (prev != static_cast<int>(wl - wf)) continue;
      __threadfence();
      if (r < nrows) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + (row0 + r) * D);
        for (int c0 = 0; c0 < D; c0 += 64) {  // 64 columns of this row at a time
          float M = -INFINITY, Ls = 0.f;
          float acc[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) acc[c] = 0.f;
          for (int64_t ww = wf; ww <= wl; ++ww) {
            const int64_t sl = ww * 2 + (si.seg_base <= tc_wstart(ww, T, W) ? 0 : 1);
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (sl * hps + r) * 2));
            const float4* src = reinterpret_cast<const float4*>(p.part_o + (sl * hps + r) * D + c0);
            float4 v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __ldcg(src + k);
            const float mn = fmaxf(M, ml.x);
            const float mu2 = (mn == -INFINITY) ? 0.f : mn;
            const float a = ptx::ex2(M - mu2), bw = ptx::ex2(ml.x - mu2);
            Ls = Ls * a + ml.y * bw;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              acc[4 * k] = acc[4 * k] * a + v[k].x * bw;
              acc[4 * k + 1] = acc[4 * k + 1] * a + v[k].y * bw;
              acc[4 * k + 2] = acc[4 * k + 2] * a + v[k].z * bw;
              acc[4 * k + 3] = acc[4 * k + 3] * a + v[k].w * bw;
            }
            M = mn;
          }
          const float iv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint4 u;
            u.x = ptx::pack_bf16x2(acc[c] * iv, acc[c + 1] * iv);
            u.y = ptx::pack_bf16x2(acc[c + 2] * iv, acc[c + 3] * iv);
            u.z = ptx::pack_bf16x2(acc[c + 4] * iv, acc[c + 5] * iv);
            u.w = ptx::pack_bf16x2(acc[c + 6] * iv, acc[c + 7] * iv);
            dst[(c0 + c) / 8] = u;
          }
        }
      }
      if (r == 0) p.counters[segid] = 0;
    }
  }

  // ---------------------------------------------------------------- exit
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 5) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
namespace {
template <int D>
constexpr size_t tc_smem_bytes() {
  using GE = TcGeo<D>;
  return 1024 + static_cast<size_t>(GE::kStages) * GE::kStage + 2 * GE::kQTile +
         GE::kStages * sizeof(TcStageInfo) + 16 * GE::kStages + 128;
}

template <int D>
cudaError_t launch_tc_t(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tq, int grid, cudaStream_t stream, bool overlap) {
  auto kern = decode_tc_kernel<D>;
  constexpr size_t smem = tc_smem_bytes<D>();
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, p);
}
}  // namespace

size_t decode_tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? tc_smem_bytes<64>() : tc_smem_bytes<128>();
}

cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tq, int grid, cudaStream_t stream, bool overlap) {
  if (p.head_dim == 64) return launch_tc_t<64>(p, tk, tv, tq, grid, stream, overlap);
  return launch_tc_t<128>(p, tk, tv, tq, grid, stream, overlap);
}

}  // namespace gqa
