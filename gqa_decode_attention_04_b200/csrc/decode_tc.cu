// Paged decode attention for large query groups (MQA-like: more than 16 query rows per K/V
// head) on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// Same result as decode_ws.cu (page "TensorRT对Multi-Query Attention的专项优化支持": decode
// re-reads all cached K/V; with MQA every query head shares one K/V head, and the plugin
// never duplicates K/V per query head; QK^T and AV run on tensor cores with K/V tiles
// prefetched into shared memory; tiny-llm "优化" page: paged KV by block table,
// FlashDecoding for long contexts).  With G query heads per K/V head the contraction is
// G flop per cached byte; for G = 96 this is a dense GEMM that CUDA-core or mma.sync code
// cannot keep up with at HBM speed, so it runs on tcgen05:
//
//   * Work list and split: as decode_ws.cu, with 64-token blocks; one contiguous range of
//     the (sequence, segment, block) list per CTA, one CTA per SM; a segment covers up to
//     128 query heads (the MMA's M = 128 rows), more heads use more segments.
//   * Producer warp: TMA copies of each block's K and V into a ring of stages (boxes of
//     the largest power of two rows dividing the page size, at most 64; a 64-row box
//     carries every column group), block-table entries read ahead through a register
//     window, and the segment's 128 query rows (one box) at each piece start.
//   * S warp (one thread issues): S_j = Q K_j^T (M = 128 heads, N = 64 tokens,
//     K = head_dim) into one of four TMEM buffers, as soon as K_j has landed and the
//     buffer's previous P V is done.
//   * P V warp (one thread issues): O_g += P_j[:, half g] V_j[half g] for the two token
//     halves, P read from TMEM, once both softmax warpgroups have written P_j.
//   * Two softmax warpgroups (256 threads; warpgroup g owns tokens [32 g, 32 g + 32) of
//     every block, thread = head row): each runs its own online softmax in the log2
//     domain over its half with its own O accumulator (rescaled in TMEM only when its
//     reference rises by more than 8), writing P (bf16) over its half of S.  At a piece
//     end the two (max, sum, O) are combined; the result is normalised and written out,
//     or, for a segment cut between CTAs, stored as a partial (O, max, sum).
//   * Split merge (a second kernel, launched with programmatic dependent launch so it is
//     resident when the decode drains): one block per cut segment and 32 rows merges the
//     partials by log-sum-exp weights.  Merging inside the decode (the last CTA of a
//     segment to finish merges it) put the merge's dependent loads behind the other CTAs'
//     K/V streams at the very end of every CTA's range.
//   * Several query tokens per sequence (the MQ instantiation, 17..128 rows per kv head):
//     a kv head's rows are its group of heads for each query token in turn (row r: token
//     r / group, head r % group), one segment per kv head.  The query tile comes from a
//     5-D tensor map (columns, head, token, column group, sequence x kv head) whose last
//     stride is group x head_dim elements, one box per column group; each softmax thread
//     masks its row's window (the sequence up to its own token) from the stage's
//     remaining length, and tile rows past the group get an empty window.
//   * 8-bit cache (the F8 instantiation): the producers copy each block's e4m3 codes into
//     a ring of raw stages; the S warp widens K (exactly) to fp16 in the tile layout its
//     MMA reads, and converts each piece's query tile from bf16 to fp16 in place, just
//     before issuing; the P V warp widens V for a block while the softmax works on it.
//     Both MMAs run kind::f16 on fp16 operands (P is packed as fp16).  The kv head's K
//     scale joins the score scale of a piece, its V scale the piece-end output.  (Two
//     extra converter warps measured slower: 14 warps cap registers at 128.)
//   * Safety: every wait is bounded; on a timeout all warps leave their loops, the MMA
//     warps wait for their issued MMAs, and TMEM is released before exit.
#include <type_traits>

#include "internal.cuh"
#include "ptx.cuh"

namespace gqa {

namespace {

constexpr int kTcBlk = 64;      // tokens per stage
constexpr int kTcRows = 128;    // MMA M: query-head rows per segment
constexpr uint32_t kTmemCols = 512;
constexpr int kTcBufs = 4;      // S/P buffers in TMEM (blocks in flight between the MMAs and the softmax)
// Warp roles: 0-7 softmax (two warpgroups, each owning half of a block's 64 tokens for all
// 128 head rows), 8 and 11 producers (even and odd blocks), 9 S MMA issuer (and TMEM
// owner), 10 P V MMA issuer.
constexpr int kTcSoftThreads = 256;
constexpr int kStgFloats = 16 * 36;  // piece-end staging per softmax warp
constexpr int kTcWarps = 12;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kWarpProducer = 8, kWarpS = 9, kWarpPV = 10, kWarpProducer2 = 11;
constexpr float kTcRescale = 8.0f;

template <int D, bool F8 = false>
struct TcGeo {
  static constexpr int kGroups = D / 64;                 // 64-column (128-byte) groups
  static constexpr int kGroupBytes = kTcBlk * 128;       // 64 rows x 128 bytes
  static constexpr int kTile = kGroups * kGroupBytes;    // K (or V) of one block (16-bit)
  static constexpr int kStage = 2 * kTile;
  static constexpr int kQGroup = kTcRows * 128;
  static constexpr int kQTile = kGroups * kQGroup;
  static constexpr int kStages = F8 ? (D == 128 ? 3 : 5) : (D == 128 ? 5 : 10);
  // 8-bit cache: a block's codes (64 tokens x D bytes per tensor, as 128-byte swizzled
  // rows) land in a ring of raw stages before the converters widen them.
  static constexpr int kRawTile = kTcBlk * D;
  static constexpr int kRawStage = 2 * kRawTile;
  static constexpr int kRawStages = F8 ? (D == 128 ? 4 : 8) : 0;
  // TMEM columns: S/P buffer k at 64 k (64 fp32 columns each; the bf16 pairs of P of
  // tokens 0-31 overwrite columns 0-15, of tokens 32-63 columns 32-47), then one O
  // accumulator (D columns) per softmax warpgroup.
  static constexpr uint32_t kO0 = 64 * kTcBufs, kO1 = kO0 + D;
  static_assert(kO1 + D <= kTmemCols, "TMEM columns");
};

struct TcStageInfo {
  uint64_t vmask;  // bit t: token t of the block is inside the sequence and its page was loaded
  int b, seg, blk, nvalid, flags, piece;
  int rem, pad;    // rem: tokens of the sequence from this block's first one on (unclamped)
};
enum : int { kTcFirst = 1, kTcLast = 2, kTcSole = 4, kTcFirstPieceOfCta = 8 };

__device__ __forceinline__ int tc_eff_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }
__device__ __forceinline__ int64_t tc_wstart(int64_t w, int64_t T, int64_t W) { return w * T / W; }
__device__ __forceinline__ int64_t tc_worker_of(int64_t x, int64_t T, int64_t W) { return ((x + 1) * W - 1) / T; }

struct TcCursor {
  int b, seg, blk, nblk, len;
};

}  // namespace

// MQ: several query tokens per sequence (p.q_len): a kv head's rows are its group of
// heads for each query token in turn (row r: token r / group, head r % group), all in one
// segment (at most 128 rows); row r sees the sequence up to its own token.
// F8: the cache holds e4m3 codes with one scale per kv head for K and for V.
template <int D, bool MQ, bool F8 = false>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                 const __grid_constant__ CUtensorMap tmap_q, const DecodeParams p) {
  using GE = TcGeo<D, F8>;
  constexpr int S = GE::kStages;
  constexpr int RS = GE::kRawStages;
  constexpr int NW = kTcWarps;
  static_assert(!(F8 && MQ), "the 8-bit cache serves one query token per sequence");
  extern __shared__ uint8_t smem_raw[];
  __shared__ int64_t s_wtot[NW];
  __shared__ float s_xmax[2][kTcRows];  // per-piece row references of each warpgroup
  __shared__ float s_xsum[2][kTcRows];  // per-piece row sums of each warpgroup
  __shared__ int s_start_b;
  __shared__ int64_t s_start_base;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  // Pieces whose query copy has been issued.  A parity wait on an mbarrier is only exact
  // if the waiter is at most one phase ahead; the two producers take pieces in turns, so
  // the one starting piece k first waits for this counter to show that piece k - 1's
  // copy was issued, which puts the barrier at most one phase behind.
  __shared__ int s_qissued;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.num_seqs;
  const int segs = p.num_kv_heads * p.n_ht;
  const int cap = p.max_blocks * p.page_size;
  const int hps = p.heads_per_seg;
  const int rows_per_seq = MQ ? p.num_heads * p.q_len : p.num_heads;

  // The split merge (the next kernel) may launch now; it waits for this grid to complete
  // before reading anything this grid writes.
  ptx::pdl_launch_dependents();
  // ---------------------------------------------------------------- prologue (split)
  int64_t mine = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = __ldg(p.seq_lens + b);
    const int Le = tc_eff_len(L, cap);
    if ((L < 0 || L > cap) && blockIdx.x == 0) atomicOr(p.err, kErrBounds);
    if (Le == 0 && (b % gridDim.x) == blockIdx.x) {
      uint32_t* o = reinterpret_cast<uint32_t*>(p.out + static_cast<int64_t>(b) * rows_per_seq * D);
      for (int i = 0; i < rows_per_seq * D / 2; ++i) o[i] = 0u;
    }
    mine += static_cast<int64_t>((Le + kTcBlk - 1) / kTcBlk) * segs;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if (lane == 0) s_wtot[warp] = mine;
  if (threadIdx.x == 0) {
    s_start_b = -1;
    s_abort = 0;
    s_qissued = 0;
  }
  __syncthreads();
  int64_t T = 0;
  for (int i = 0; i < NW; ++i) T += s_wtot[i];
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
      for (int i = 0; i < NW; ++i) {
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
  const uint32_t raw = ring + S * GE::kStage;               // F8: RS raw stages of K | V codes
  const uint32_t qbuf = raw + RS * GE::kRawStage;           // Q tile of the current piece
  uint8_t* vring = base_ptr;                                // generic view of the ring
  TcStageInfo* info = reinterpret_cast<TcStageInfo*>(base_ptr + S * GE::kStage + RS * GE::kRawStage + GE::kQTile);
  TcStageInfo* rinfo = info + S;                            // F8: descriptors of the raw stages
  const uint32_t bar0 = ptx::smem_u32(rinfo + RS);
  const uint32_t full_bar = bar0;                 // [S] producer -> MMA (K/V landed)
  const uint32_t empty_bar = full_bar + 8 * S;    // [S] MMA commit -> producer
  const uint32_t qfull_bar = empty_bar + 8 * S;   // producer -> S warp (piece k: phase k)
  const uint32_t qempty_bar = qfull_bar + 8;      // S warp commit -> producer
  const uint32_t sfull_bar = qempty_bar + 8;             // [kTcBufs] S warp commit -> softmax
  const uint32_t pfull_bar = sfull_bar + 8 * kTcBufs;    // [kTcBufs] softmax (256) -> P V warp
  const uint32_t pv_bar = pfull_bar + 8 * kTcBufs;       // [kTcBufs] P V warp commit after block j's P V
  const uint32_t ofree_bar = pv_bar + 8 * kTcBufs;       // softmax (256) -> P V warp, a piece's O is read
  const uint32_t drain_bar = ofree_bar + 8;       // MMA commit at exit
  const uint32_t wg_bar = drain_bar + 8;          // rendezvous of both softmax warpgroups (256)
  const uint32_t raw_full = wg_bar + 8;           // F8: [RS] producer -> S and P V warps (codes landed)
  const uint32_t raw_empty = raw_full + 8 * RS;   // F8: [RS] S warp (K) and P V warp (V) converted -> producer
  const uint32_t bars_end = raw_empty + 8 * RS;
  // Piece-end staging: per softmax warp 16 rows x 36 floats, so a warp writes whole
  // 128-byte row segments of its 32 rows (16 rows per round) instead of one row per lane.
  float* const stg_all = reinterpret_cast<float*>(base_ptr + ((bars_end - ring + 127u) & ~127u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar + 8 * s, 1);
      ptx::mbar_init(empty_bar + 8 * s, 1);
    }
    ptx::mbar_init(qfull_bar, 1);
    ptx::mbar_init(qempty_bar, 1);
    for (int k = 0; k < kTcBufs; ++k) {
      ptx::mbar_init(sfull_bar + 8 * k, 1);
      ptx::mbar_init(pfull_bar + 8 * k, kTcSoftThreads);
      ptx::mbar_init(pv_bar + 8 * k, 1);
    }
    ptx::mbar_init(ofree_bar, kTcSoftThreads);
    ptx::mbar_init(drain_bar, 2);  // both MMA-issuing warps
    ptx::mbar_init(wg_bar, kTcSoftThreads);
    if constexpr (F8) {
      for (int s = 0; s < RS; ++s) {
        ptx::mbar_init(raw_full + 8 * s, 1);
        ptx::mbar_init(raw_empty + 8 * s, 2);
      }
    }
    ptx::fence_mbarrier_init();
  }
  if (warp == kWarpS) ptx::tmem_alloc(ptx::smem_u32(&s_tmem), kTmemCols);
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
  // 8-bit cache: one warp widens one tensor's codes of a block (raw stage, 128-byte
  // swizzled rows) into the 16-bit tile its MMA reads ([group][64 rows][128 B], swizzled).
  // Lane (t, c): 8 lanes take 8 tokens of one 16-code chunk, so the swizzled reads and
  // writes hit distinct banks.
  auto convert_tile = [&](uint32_t raw_tile, uint32_t tile) {
    constexpr int CPT = D / 16;               // 16-code chunks per token
    constexpr int ITERS = kTcBlk * CPT / 32;  // chunks per lane
    constexpr int BATCH = 8;                  // chunks loaded before any is converted (latency)
    const uint8_t* rb = base_ptr + (raw_tile - ring);
    uint8_t* fb = base_ptr + (tile - ring);
    const int tlo = lane & 7, cq = lane >> 3;
#pragma unroll
    for (int i0 = 0; i0 < ITERS; i0 += BATCH) {
      uint4 x[BATCH];
#pragma unroll
      for (int j = 0; j < BATCH; ++j) {
        const int it = i0 + j;
        const int c = cq + 4 * (it % (CPT / 4));  // head dims 16 c .. 16 c + 15
        const int tok = 8 * (it / (CPT / 4)) + tlo;
        const int rrow = tok / (128 / D);
        const int rc = (tok % (128 / D)) * CPT + c;
        x[j] = *reinterpret_cast<const uint4*>(rb + rrow * 128 + ((rc ^ (rrow & 7)) << 4));
      }
#pragma unroll
      for (int j = 0; j < BATCH; ++j) {
        const int it = i0 + j;
        const int c = cq + 4 * (it % (CPT / 4));
        const int tok = 8 * (it / (CPT / 4)) + tlo;
        const int cc = 2 * (c % 4);  // 8-value chunk of its 64-column group
        uint8_t* dst = fb + (c / 4) * GE::kGroupBytes + tok * 128;
        *reinterpret_cast<uint4*>(dst + ((cc ^ (tok & 7)) << 4)) =
            make_uint4(ptx::e4m3x2_lo(x[j].x), ptx::e4m3x2_hi(x[j].x), ptx::e4m3x2_lo(x[j].y), ptx::e4m3x2_hi(x[j].y));
        *reinterpret_cast<uint4*>(dst + (((cc + 1) ^ (tok & 7)) << 4)) =
            make_uint4(ptx::e4m3x2_lo(x[j].z), ptx::e4m3x2_hi(x[j].z), ptx::e4m3x2_lo(x[j].w), ptx::e4m3x2_hi(x[j].w));
      }
    }
  };

  if (warp == kWarpProducer || warp == kWarpProducer2) {
    // ============================================================ producer warps
    // Both walk every 64-token block of the range; producer `pid` issues the blocks with
    // i % 2 == pid (its stage descriptor, copy barrier, K/V copies, and the piece's Q copy
    // when the block starts a piece), so the serial per-block issue work is split in two.
    // The loop carries no integer division and no 64-bit index arithmetic: page positions
    // advance incrementally and divisions happen once per piece.
    const uint32_t pid = warp == kWarpProducer ? 0u : 1u;
    if (lane == 0) {
      ptx::prefetch_tensormap(&tmap_k);
      ptx::prefetch_tensormap(&tmap_v);
      ptx::prefetch_tensormap(&tmap_q);
    }
    const uint64_t policy = ptx::policy_evict_first();
    const int ps = p.page_size;
    const int R = tc_box_rows(ps);           // rows per TMA box: divides both 64 and ps
    const int nchunks = kTcBlk / R;          // boxes (page pieces) per block and tensor
    // A 64-row box carries every 64-column group at once (its shared-memory image is the
    // [group][64 rows][128 B] tile the MMAs read); shorter boxes carry one group each.
    const int box_groups = R == kTcBlk ? GE::kGroups : 1;
    // (8-bit cache: one box of R * D / 128 code rows carries a chunk's every column)
    const int gsteps = F8 ? 1 : GE::kGroups / box_groups;
    const int nops = 2 * nchunks * gsteps;   // copies per block, one per lane
    // This lane's copy: tensor (K or V), chunk and column group.
    const int op_t = lane / (nchunks * gsteps);
    const int op_c = (lane % (nchunks * gsteps)) / gsteps;
    const int op_g = (lane % gsteps) * box_groups;
    const int cl = lane & (nchunks - 1);     // chunk whose page this lane tracks
    const uint32_t tile_bytes = F8 ? 2u * R * D : 2u * GE::kGroups * R * 128u;  // K + V bytes of one chunk
    // The ring the copies land in: the MMA stages, or with the 8-bit cache the raw ones.
    constexpr int PS = F8 ? RS : S;
    const uint32_t p_full = F8 ? raw_full : full_bar;
    const uint32_t p_empty = F8 ? raw_empty : empty_bar;
    TcStageInfo* const p_info = F8 ? rinfo : info;
    // Block-table rows are read 32 entries at a time (one per lane) into a register window,
    // with the window needed next already in flight, so no copy waits on a dependent load.
    // Window boundaries (entry 32 k starts at token 32 k ps, a multiple of 512) fall on
    // block boundaries, so one block's entries share a window.
    auto load_window = [&](int b, int k) -> int {
      const int e = 32 * k + lane;
      return (b >= 0 && b < B && e < p.max_blocks)
                 ? __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + e) : -1;
    };
    int wb = -1, wk = -1, wval = -1;  // window in use: row wb, entries [32 wk, 32 wk + 32)
    int nb = -1, nk = -1, nval = -1;  // window prefetched next
    int next_len = (cu.b + 1 < B) ? __ldg(p.seq_lens + cu.b + 1) : 0;
    // Chunk cl of the cursor's block starts at token t = 64 blk + cl R: block-table entry
    // pe = t / ps, row po = t % ps inside that page.
    int pe = 0, po = 0, kvh = 0, ht = 0, q_row0 = 0;
    auto start_piece = [&]() {
      const int t = cu.blk * kTcBlk + cl * R;
      pe = t / ps;
      po = t - pe * ps;
      kvh = cu.seg / p.n_ht;
      ht = cu.seg - kvh * p.n_ht;
      q_row0 = cu.b * p.num_heads + kvh * p.group + ht * hps;
    };
    auto page_of = [&]() -> int {  // this lane's chunk page, -1 past the sequence end
      const int k = pe >> 5;
      if (cu.b != wb || k != wk) {
        wval = (cu.b == nb && k == nk) ? nval : load_window(cu.b, k);
        wb = cu.b;
        wk = k;
        const int entries = (cu.len + ps - 1) / ps;
        if (32 * (k + 1) < entries) { nb = cu.b; nk = k + 1; }
        else if (cu.seg + 1 < segs) { nb = cu.b; nk = 0; }
        else { nb = cu.b + 1; nk = 0; }
        nval = load_window(nb, nk);
      }
      const int pg = __shfl_sync(0xffffffffu, wval, pe & 31);
      return (lane < nchunks && cu.blk * kTcBlk + cl * R < cu.len) ? pg : -1;
    };
    start_piece();
    int piece = 0;
    bool first_piece = true;
    int piece_blk0 = cu.blk;
    int page = page_of();
    int stage = 0;
    uint32_t round = 0;  // times the ring has wrapped
    int64_t i = 0;
    ptx::pdl_wait_prerequisites();  // K/V pools may be written by the previous kernel
    for (; i < total; ++i) {
      const bool mine = (static_cast<uint32_t>(i) & 1u) == pid;
      const bool first = (i == 0) || cu.blk == 0;
      const bool last = (i + 1 == total) || (cu.blk + 1 == cu.nblk);
      if (first) piece_blk0 = cu.blk;
      if (mine) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      if (round > 0) {
        const bool ok = ptx::mbar_wait_bounded(p_empty + 8 * stage, (round - 1) & 1u, limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
      }
      if (first) {
        // Q rows of this piece's segment (the previous piece's S MMAs must be done with it).
        // Piece - 1's copy was issued only after the phase of piece - 2 completed, so once
        // it has been issued the parity wait can only be met by the phase of piece - 1.
        bool ok = true;
        if (piece >= 1) {
          ok = ptx::wait_counter(&s_qissued, piece, limit);
          if (ok) ok = ptx::mbar_wait_bounded(qempty_bar, static_cast<uint32_t>((piece - 1) & 1), limit);
        }
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
        if (lane == 0) {
          if constexpr (MQ) {
            // One box per column group: the kv head's rows (token, head) of this sequence
            // (the 5-D map: columns, head, token, column group, sequence x kv head).
            const uint32_t qbytes = static_cast<uint32_t>(p.group) * p.q_len * D * 2u;
            ptx::mbar_arrive_expect_tx(qfull_bar, p.arm_without_copy ? 1u : qbytes);
            if (!p.arm_without_copy)
              for (int cgi = 0; cgi < GE::kGroups; ++cgi)
                ptx::tma_load_5d(qbuf + cgi * GE::kQGroup, &tmap_q, qfull_bar, 0, 0, 0, cgi,
                                 (cu.b * p.q_len) * p.num_kv_heads + kvh);
          } else {
            ptx::mbar_arrive_expect_tx(qfull_bar, p.arm_without_copy ? 1u : GE::kQTile);
            if (!p.arm_without_copy)  // one box: 128 rows x every column group
              ptx::tma_load_3d(qbuf, &tmap_q, qfull_bar, 0, q_row0, 0, 0);
          }
          *reinterpret_cast<volatile int*>(&s_qissued) = piece + 1;
        }
      }
      const int nvalid = min(kTcBlk, cu.len - cu.blk * kTcBlk);
      const bool want = lane < nchunks && lane * R < nvalid;
      const bool ok = want && page >= 0 && page < p.num_pages;
      const uint32_t wantbits = __ballot_sync(0xffffffffu, want);
      const uint32_t okbits = __ballot_sync(0xffffffffu, ok);
      const int op_page = __shfl_sync(0xffffffffu, page, op_c);
      const int op_po = __shfl_sync(0xffffffffu, po, op_c);
      if (lane == 0) {
        if (wantbits != okbits) atomicOr(p.err, kErrBounds);
        uint64_t vmask = 0;
        const uint64_t chunk_mask = R >= 64 ? ~0ull : ((1ull << R) - 1ull);
        for (int c = 0; c < nchunks; ++c)
          if ((okbits >> c) & 1u) vmask |= chunk_mask << (c * R);
        if (nvalid < kTcBlk) vmask &= (1ull << nvalid) - 1ull;
        TcStageInfo& si = p_info[stage];
        si.vmask = vmask;
        si.b = cu.b;
        si.seg = cu.seg;
        si.blk = cu.blk;
        si.nvalid = nvalid;
        si.rem = cu.len - cu.blk * kTcBlk;
        si.piece = piece;
        si.flags = (first ? kTcFirst : 0) | (last ? kTcLast : 0) |
                   ((last && piece_blk0 == 0 && cu.blk + 1 == cu.nblk) ? kTcSole : 0) |
                   (first_piece ? kTcFirstPieceOfCta : 0);
        const uint32_t bytes = p.arm_without_copy ? 0u : __popc(okbits) * tile_bytes;
        if (bytes) ptx::mbar_arrive_expect_tx(p_full + 8 * stage, bytes);
        else if (p.arm_without_copy) ptx::mbar_arrive_expect_tx(p_full + 8 * stage, 1u);
        else ptx::mbar_arrive(p_full + 8 * stage);
      }
      __syncwarp();
      if (lane < nops && ((okbits >> op_c) & 1u) && !p.arm_without_copy) {
        const int row = (op_page * p.num_kv_heads + kvh) * ps + op_po;
        if constexpr (F8) {  // codes: R tokens are R * D / 128 rows of 128 bytes
          const uint32_t dst = raw + stage * GE::kRawStage + op_t * GE::kRawTile + op_c * R * D;
          ptx::tma_load_2d(dst, op_t ? &tmap_v : &tmap_k, p_full + 8 * stage, 0, row / (128 / D), policy);
        } else {
          const uint32_t dst = ring + stage * GE::kStage + op_t * GE::kTile + op_g * GE::kGroupBytes + op_c * R * 128;
          ptx::tma_load_3d(dst, op_t ? &tmap_v : &tmap_k, full_bar + 8 * stage, 0, row, op_g, policy);
        }
      }
      }  // mine
      if (++stage == PS) {
        stage = 0;
        ++round;
      }
      if (last) {
        first_piece = false;
        ++piece;
      }
      if (i + 1 < total) {
        if (++cu.blk < cu.nblk) {
          po += kTcBlk;  // next block of the same piece
          while (po >= ps) {
            po -= ps;
            ++pe;
          }
        } else {
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
          start_piece();
        }
        page = page_of();
      }
    }
    // Let this producer's copies still in flight land before the CTA can exit.
    for (int64_t j = (i > PS ? i - PS : 0); j < i; ++j)
      if ((static_cast<uint32_t>(j) & 1u) == pid)
        ptx::mbar_wait_bounded(p_full + 8 * (j % PS), static_cast<uint32_t>((j / PS) & 1), limit);
  } else if (warp == kWarpS) {
    // ============================================================ S warp
    // S_n = Q K_n^T into TMEM buffer n % kTcBufs once block n's K has landed and the P V of
    // block n - kTcBufs (issued by the P V warp, reading P from the same buffer) is complete.
    constexpr uint32_t idS = F8 ? ptx::umma_idesc_f16(kTcRows, kTcBlk, false) : ptx::umma_idesc_bf16(kTcRows, kTcBlk, false);
    bool issued = false;  // a tcgen05.commit is only used to track MMAs this warp issued
    for (int64_t n = 0; n < total; ++n) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      const int stage = static_cast<int>(n % S);
      bool ok;
      TcStageInfo si;
      if constexpr (F8) {
        // Block n's codes have landed and the stage's previous block is consumed (its P V is
        // complete); at a piece start also the piece's Q copy (pieces in order: exact parity).
        const int rst = static_cast<int>(n % RS);
        ok = ptx::mbar_wait_bounded(raw_full + 8 * rst, static_cast<uint32_t>((n / RS) & 1), limit);
        if (ok && n >= S) ok = ptx::mbar_wait_bounded(empty_bar + 8 * stage, static_cast<uint32_t>((n / S - 1) & 1), limit);
        si = rinfo[rst];
        if (ok && (si.flags & kTcFirst)) ok = ptx::mbar_wait_bounded(qfull_bar, static_cast<uint32_t>(si.piece & 1), limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
        if (si.flags & kTcFirst) {  // the piece's query tile, bf16 -> fp16 in place
          uint4* qv = reinterpret_cast<uint4*>(base_ptr + (qbuf - ring));
          for (int k = lane; k < GE::kQTile / 16; k += 32) {
            uint4 x = qv[k];
            x.x = ptx::bf16x2_to_f16x2(x.x);
            x.y = ptx::bf16x2_to_f16x2(x.y);
            x.z = ptx::bf16x2_to_f16x2(x.z);
            x.w = ptx::bf16x2_to_f16x2(x.w);
            qv[k] = x;
          }
        }
        convert_tile(raw + rst * GE::kRawStage, ring + stage * GE::kStage);
        if (lane == 0) {
          info[stage] = si;
          __threadfence_block();
        }
        ptx::fence_proxy_async_smem();  // the MMA reads the converted tiles through the async proxy
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(raw_empty + 8 * rst);
        if (n >= kTcBufs)
          ok = ptx::mbar_wait_bounded(pv_bar + 8 * (n % kTcBufs),
                                      static_cast<uint32_t>(((n - kTcBufs) / kTcBufs) & 1), limit);
      } else {
        ok = ptx::mbar_wait_bounded(full_bar + 8 * stage, static_cast<uint32_t>((n / S) & 1), limit);
        si = info[stage];
        if (ok && (si.flags & kTcFirst))
          ok = ptx::mbar_wait_bounded(qfull_bar, static_cast<uint32_t>(si.piece & 1), limit);
        if (ok && n >= kTcBufs)
          ok = ptx::mbar_wait_bounded(pv_bar + 8 * (n % kTcBufs),
                                      static_cast<uint32_t>(((n - kTcBufs) / kTcBufs) & 1), limit);
      }
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) abort_all(kErrTimeout);
        break;
      }
      ptx::tc_fence_after();
      if (lane == 0) {
        const int sb = static_cast<int>(n % kTcBufs);
        const uint32_t kb = ring + stage * GE::kStage;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t a = ptx::umma_desc_sw128(qbuf + (ks >> 2) * GE::kQGroup + (ks & 3) * 32, 16, 1024);
          const uint64_t b = ptx::umma_desc_sw128(kb + (ks >> 2) * GE::kGroupBytes + (ks & 3) * 32, 16, 1024);
          ptx::umma_ss(tmem + 64 * sb, a, b, idS, ks > 0 ? 1u : 0u);
        }
        ptx::umma_commit(sfull_bar + 8 * sb);
        if (si.flags & kTcLast) ptx::umma_commit(qempty_bar);  // Q tile no longer read
      }
      issued = true;
      __syncwarp();
    }
    // Every MMA issued by this warp completes before TMEM can be released.  A warp that
    // issued none (its first wait ran out) arrives directly.
    if (lane == 0) {
      if (issued) ptx::umma_commit(drain_bar);
      else ptx::mbar_arrive(drain_bar);
    }
    __syncwarp();
    ptx::mbar_wait_bounded(drain_bar, 0, limit);
  } else if (warp == kWarpPV) {
    // ============================================================ P V warp
    // O += P_m V_m as soon as the softmax has written P_m (and, at a piece start, has read
    // the previous piece's O out).
    constexpr uint32_t idPV = F8 ? ptx::umma_idesc_f16(kTcRows, D, true) : ptx::umma_idesc_bf16(kTcRows, D, true);
    bool issued = false;
    for (int64_t m = 0; m < total; ++m) {
      if (__any_sync(0xffffffffu, aborted())) break;  // warp-uniform
      const int k = static_cast<int>(m % kTcBufs);
      const int stage = static_cast<int>(m % S);
      bool ok;
      if constexpr (F8) {
        // Widen V_m while the softmax works on block m: its codes have landed and this
        // warp's P V of the stage's previous block is complete.
        const int rst = static_cast<int>(m % RS);
        ok = ptx::mbar_wait_bounded(raw_full + 8 * rst, static_cast<uint32_t>((m / RS) & 1), limit);
        if (ok && m >= S) ok = ptx::mbar_wait_bounded(empty_bar + 8 * stage, static_cast<uint32_t>((m / S - 1) & 1), limit);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) abort_all(kErrTimeout);
          break;
        }
        convert_tile(raw + rst * GE::kRawStage + GE::kRawTile, ring + stage * GE::kStage + GE::kTile);
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(raw_empty + 8 * rst);
        ok = ptx::mbar_wait_bounded(pfull_bar + 8 * k, static_cast<uint32_t>((m / kTcBufs) & 1), limit);
      } else {
        ok = ptx::mbar_wait_bounded(pfull_bar + 8 * k, static_cast<uint32_t>((m / kTcBufs) & 1), limit);
        // V_m landed before S_m was issued; observing the copy barrier here as well orders
        // the TMA writes before this warp's own stores and MMAs (it has already completed).
        if (ok) ok = ptx::mbar_wait_bounded(full_bar + 8 * stage, static_cast<uint32_t>((m / S) & 1), limit);
      }
      const TcStageInfo si = info[stage];  // the stage is held until this P V completes
      const bool first = si.flags & kTcFirst;
      if (ok && first && si.piece > 0)
        ok = ptx::mbar_wait_bounded(ofree_bar, static_cast<uint32_t>((si.piece - 1) & 1), limit);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) abort_all(kErrTimeout);
        break;
      }
      if (si.vmask != ~0ull) {
        // Rows of tokens past the sequence end (or of pages that failed the range check)
        // may hold any bits, NaN included: zero them in V so 0 * NaN cannot reach O.
        // (Their scores are masked to -inf by the softmax.)
        uint8_t* v = vring + stage * GE::kStage + GE::kTile;
        for (int idx = lane; idx < kTcBlk * 8 * GE::kGroups; idx += 32) {
          const int g = idx / (kTcBlk * 8);
          const int r = (idx / 8) % kTcBlk, c = idx % 8;
          if (!((si.vmask >> r) & 1ull))
            *reinterpret_cast<uint4*>(v + g * GE::kGroupBytes + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
      }
      ptx::tc_fence_after();
      if (lane == 0) {
        const uint32_t vb = ring + stage * GE::kStage + GE::kTile;
        const uint32_t pt = tmem + 64 * k;
#pragma unroll
        for (int ks = 0; ks < kTcBlk / 16; ++ks) {
          const uint64_t bdesc = ptx::umma_desc_sw128(vb + ks * 16 * 128, GE::kGroupBytes, 1024);
          // Tokens 0-31 accumulate into warpgroup 0's O, tokens 32-63 into warpgroup 1's;
          // P of tokens 16 ks .. 16 ks + 15 sits at column 32 (ks / 2) + 8 (ks % 2).
          ptx::umma_ts(tmem + (ks < 2 ? GE::kO0 : GE::kO1), pt + (ks >> 1) * 32 + (ks & 1) * 8, bdesc,
                       idPV, (first && (ks & 1) == 0) ? 0u : 1u);
        }
        ptx::umma_commit(empty_bar + 8 * stage);  // K_m and V_m are consumed
        ptx::umma_commit(pv_bar + 8 * k);
      }
      issued = true;
      __syncwarp();
    }
    if (lane == 0) {
      if (issued) ptx::umma_commit(drain_bar);
      else ptx::mbar_arrive(drain_bar);
    }
    __syncwarp();
    ptx::mbar_wait_bounded(drain_bar, 0, limit);
  } else {
    // ============================================================ softmax warpgroups
    // Thread t: warpgroup g = t / 128 owns tokens [32 g, 32 g + 32) of every block and its
    // own O accumulator in TMEM; row r = t % 128 is query head r of the segment tile
    // (TMEM lane r).  The two warpgroups run independent online softmaxes over their
    // halves (no per-block exchange) and combine the two (max, sum, O) at a piece end.
    const int t = threadIdx.x;
    const int g = t >> 7, r = t & (kTcRows - 1);
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t o_mine = tmem + lane_off + (g ? GE::kO1 : GE::kO0);
    float sl2 = p.scale_log2;     // (8-bit cache: times the kv head's K scale, set per piece)
    bool pos = sl2 >= 0.f;        // a negative scale turns the row maximum into a minimum
    constexpr int HD = D / 2;     // output columns each warpgroup finishes at a piece end
    float mref = -INFINITY, lsum = 0.f;
    // MQ: query tokens newer than this row's own.  Rows past the group's are padding whose
    // query rows are stale shared memory: their window is empty, so they never trigger an
    // O rescale (which waits for every earlier P V) and contribute nothing.
    const int cdrop = MQ ? (r < p.group * p.q_len ? p.q_len - 1 - r / p.group : (1 << 30)) : 0;
    int wg_phase = 0;
    bool failed = false;
    // Every wait outcome is made warp-uniform: the TMEM loads and stores that follow are
    // warp-collective (.sync.aligned) and must never run on part of a warp.
    // P V MMAs are issued by one thread and complete in order, so "the P V of block j is
    // complete" (phase j / kTcBufs of pv_bar[j % kTcBufs]) covers every earlier block.  It
    // is only waited for at block i with j >= i - 1: the barrier's next phase (block
    // j + kTcBufs) needs a P this warpgroup has not written yet, so parity is unambiguous.
    auto wait_pv_done = [&](int64_t j) -> bool {
      const bool ok = ptx::mbar_wait_bounded(pv_bar + 8 * (j % kTcBufs),
                                             static_cast<uint32_t>((j / kTcBufs) & 1), limit);
      return __all_sync(0xffffffffu, ok);
    };
    auto wg_sync = [&]() -> bool {  // all 256 softmax threads (bounded)
      ptx::mbar_arrive(wg_bar);
      const bool ok = ptx::mbar_wait_bounded(wg_bar, static_cast<uint32_t>(wg_phase & 1), limit);
      ++wg_phase;
      return __all_sync(0xffffffffu, ok);
    };
    int is = 0;  // stage of block i (i % S, kept incrementally)
    for (int64_t i = 0; i < total && !failed; ++i) {
      // Another warp's failed wait ends the CTA; checked every 8 blocks (each wait here is
      // bounded, so a stale flag only costs time).
      const uint32_t i32 = static_cast<uint32_t>(i);  // buffer / phase arithmetic mod 2^32
      if ((i32 & 7u) == 0 && __any_sync(0xffffffffu, aborted())) break;
      const int sb = static_cast<int>(i32 % kTcBufs);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(sfull_bar + 8 * sb, (i32 / kTcBufs) & 1u, limit))) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      const int stg = is;
      if (++is == S) is = 0;
      const TcStageInfo* const ip = &info[stg];
      const int flags = ip->flags;
      const uint64_t vmask = ip->vmask;
      // What a piece end needs of this block, read while its stage is held (the stage is
      // refilled once the block's P V completes, which needs this thread's P).
      int pe_b = 0, pe_seg = 0;
      if (flags & kTcLast) {
        pe_b = ip->b;
        pe_seg = ip->seg;
      }
      const bool first = flags & kTcFirst;
      if (first) {
        mref = -INFINITY;
        lsum = 0.f;
        if constexpr (F8) {
          sl2 = p.scale_log2 * __ldg(p.k_scales + ip->seg / p.n_ht);
          pos = sl2 >= 0.f;
        }
      }
      const uint32_t st = tmem + lane_off + 64 * sb;
      uint32_t u[32];
      ptx::tmem_ld32(st + 32 * g, u);
      ptx::tmem_wait_ld();
      // Scores of tokens outside the sequence (or of pages that failed the range check)
      // may be anything, NaN included: they take the raw value that scales to -inf.
      uint32_t vm = static_cast<uint32_t>(vmask >> (32 * g));
      if constexpr (MQ) {  // this row's window ends q_len - 1 - (its token) tokens early
        const int lim = info[stg].rem - cdrop - 32 * g;
        if (lim < 32) vm &= lim <= 0 ? 0u : ((1u << lim) - 1u);
      }
      const bool full = vm == 0xffffffffu;
      if (!full) {
        const uint32_t off = pos ? 0xff800000u : 0x7f800000u;  // -inf / +inf
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (!((vm >> c) & 1u)) u[c] = off;
      }
      // Row maximum of this half's scaled scores (log2 domain), a tree over raw scores.
      float mx;
      {
        // 32 -> 11 -> 4 -> 1 with three-input max (min for a negative scale).
        float tt[11];
        if (pos) {
#pragma unroll
          for (int c = 0; c < 10; ++c)
            tt[c] = ptx::max3(__uint_as_float(u[3 * c]), __uint_as_float(u[3 * c + 1]), __uint_as_float(u[3 * c + 2]));
          tt[10] = fmaxf(__uint_as_float(u[30]), __uint_as_float(u[31]));
          tt[0] = ptx::max3(tt[0], tt[1], tt[2]);
          tt[3] = ptx::max3(tt[3], tt[4], tt[5]);
          tt[6] = ptx::max3(tt[6], tt[7], tt[8]);
          tt[9] = fmaxf(tt[9], tt[10]);
          tt[0] = fmaxf(ptx::max3(tt[0], tt[3], tt[6]), tt[9]);
        } else {
#pragma unroll
          for (int c = 0; c < 10; ++c)
            tt[c] = ptx::min3(__uint_as_float(u[3 * c]), __uint_as_float(u[3 * c + 1]), __uint_as_float(u[3 * c + 2]));
          tt[10] = fminf(__uint_as_float(u[30]), __uint_as_float(u[31]));
          tt[0] = ptx::min3(tt[0], tt[1], tt[2]);
          tt[3] = ptx::min3(tt[3], tt[4], tt[5]);
          tt[6] = ptx::min3(tt[6], tt[7], tt[8]);
          tt[9] = fminf(tt[9], tt[10]);
          tt[0] = fminf(ptx::min3(tt[0], tt[3], tt[6]), tt[9]);
        }
        mx = tt[0] * sl2;
        if (mx != mx) mx = -INFINITY;  // every token masked and a zero scale
      }
      const bool need = mx > mref + kTcRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ptx::ex2(mref - mx) : 1.f;  // 0 when mref = -inf
        if (!first) {
          // Rescale this warpgroup's O rows in TMEM once every earlier P V is in.  The
          // whole warp takes part; rows that keep their reference scale by 1.
          if (!wait_pv_done(i - 1)) {
            abort_all(kErrTimeout);
            failed = true;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            ptx::tmem_ld32(o_mine + c0, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            ptx::tmem_st32(o_mine + c0, ov);
          }
          ptx::tmem_wait_st();
        }
        if (need) {
          lsum *= alpha;
          mref = mx;
        }
      }
      // P = 2^(score * scale_log2 - reference), one ex2 per score (the arguments and the
      // row sum in packed fp32 pairs, two scores per instruction); bf16
      // pairs overwrite the first 16 of this half's own 32 score columns (token 32 g + 2j,
      // 32 g + 2j + 1 in column 32 g + j), so neither warpgroup touches the other's scores.
      const float nmu = (mref == -INFINITY) ? 0.f : -mref;
      // Three passes (arguments, exponentials, sums and packing) so the 32 ex2 issue back
      // to back on the MUFU.
      float e[32];
      {
        const uint64_t s2 = ptx::f2_pack(sl2, sl2), n2 = ptx::f2_pack(nmu, nmu);
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(u[c]), __uint_as_float(u[c + 1])), s2, n2),
                         e[c], e[c + 1]);
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) e[c] = ptx::ex2(e[c]);
      if (!full) {  // masked scores are exactly 0 (with a zero scale, inf * 0 is NaN)
#pragma unroll
        for (int c = 0; c < 32; ++c) e[c] = ((vm >> c) & 1u) ? e[c] : 0.f;
      }
      uint32_t pk[16];
      {
        uint64_t a0 = ptx::f2_pack(e[0], e[1]), a1 = ptx::f2_pack(e[2], e[3]);
#pragma unroll
        for (int c = 4; c < 32; c += 4) {
          a0 = ptx::f2_add(a0, ptx::f2_pack(e[c], e[c + 1]));
          a1 = ptx::f2_add(a1, ptx::f2_pack(e[c + 2], e[c + 3]));
        }
        float s0, s1;
        ptx::f2_unpack(ptx::f2_add(a0, a1), s0, s1);
        lsum += s0 + s1;
      }
#pragma unroll
      for (int c = 0; c < 32; c += 2) pk[c / 2] = F8 ? ptx::pack_f16x2(e[c], e[c + 1]) : ptx::pack_bf16x2(e[c], e[c + 1]);
      ptx::tmem_st16(st + 32 * g, pk);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(pfull_bar + 8 * sb);

      if (!(flags & kTcLast)) continue;
      // ---------------------------------------------------------- end of a piece
      // Combine the two halves: M = max(m0, m1), O = sum_g O_g 2^(m_g - M),
      // L = sum_g l_g 2^(m_g - M).  Warpgroup g finishes output columns [g HD, g HD + HD).
      if (!wait_pv_done(i)) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      ptx::tc_fence_after();
      s_xmax[g][r] = mref;
      s_xsum[g][r] = lsum;
      if (!wg_sync()) {
        abort_all(kErrTimeout);
        failed = true;
        break;
      }
      const float m0 = s_xmax[0][r], m1 = s_xmax[1][r];
      const float Mx = fmaxf(m0, m1);
      const float Mu = (Mx == -INFINITY) ? 0.f : Mx;
      const float w0 = ptx::ex2(m0 - Mu), w1 = ptx::ex2(m1 - Mu);  // 0 for an empty half
      const float ltot = s_xsum[0][r] * w0 + s_xsum[1][r] * w1;
      const int kvh = pe_seg / p.n_ht, ht = pe_seg % p.n_ht;
      const int nrows = min(hps, (MQ ? p.group * p.q_len : p.group) - ht * hps);
      const int64_t row0 = static_cast<int64_t>(pe_b) * p.num_heads + kvh * p.group + ht * hps;
      const bool sole = flags & kTcSole;
      const int64_t slot = w * 2 + ((flags & kTcFirstPieceOfCta) ? 0 : 1);
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      float f0 = sole ? w0 * inv : w0, f1 = sole ? w1 * inv : w1;
      if constexpr (F8) {  // cached V values are codes x the kv head's V scale
        const float vs = __ldg(p.v_scales + kvh);
        f0 *= vs;
        f1 *= vs;
      }
      float* const rows_buf = stg_all + warp * kStgFloats;
#pragma unroll
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t oa[32], ob[32];
        ptx::tmem_ld32(tmem + lane_off + GE::kO0 + g * HD + c0, oa);
        ptx::tmem_ld32(tmem + lane_off + GE::kO1 + g * HD + c0, ob);
        ptx::tmem_wait_ld();
        float* o = reinterpret_cast<float*>(oa);  // combined in place (constant indices only)
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(oa[c]) * f0 + __uint_as_float(ob[c]) * f1;
        // 16 rows at a time through shared memory: lane l then writes 4 columns of row
        // (l / 8) + 4m, so 8 lanes cover one 128-byte row segment.
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          if ((lane >> 4) == rr) {
            float4* w4 = reinterpret_cast<float4*>(rows_buf + (lane & 15) * 36);
#pragma unroll
            for (int c = 0; c < 8; ++c) w4[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          }
          __syncwarp();
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int lr = (lane >> 3) + 4 * m;
            const int row = 32 * (warp & 3) + 16 * rr + lr;  // row of the segment tile
            const float4 x = *reinterpret_cast<const float4*>(rows_buf + lr * 36 + (lane & 7) * 4);
            const int col = g * HD + c0 + (lane & 7) * 4;
            if (row < nrows) {
              if (sole) {  // out is only 8-byte aligned: 4 columns per store
                uint2 v;
                v.x = ptx::pack_bf16x2(x.x, x.y);
                v.y = ptx::pack_bf16x2(x.z, x.w);
                const int64_t orow =
                    MQ ? (static_cast<int64_t>(pe_b) * p.q_len + row / p.group) * p.num_heads + kvh * p.group +
                             row % p.group
                       : row0 + row;
                *reinterpret_cast<uint2*>(p.out + orow * D + col) = v;
              } else {
                *reinterpret_cast<float4*>(p.part_o + (slot * hps + row) * D + col) = x;
              }
            }
          }
          __syncwarp();
        }
      }
      if (!sole && g == 0 && r < nrows)
        *reinterpret_cast<float2*>(p.part_ml + (slot * hps + r) * 2) = make_float2(Mx, ltot);
      ptx::tc_fence_before();
      ptx::mbar_arrive(ofree_bar);  // O may be overwritten by the next piece
    }
  }

  // ---------------------------------------------------------------- exit
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kWarpS) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ split merge
// Second kernel of a tcgen05 decode.  Block (w - 1, y) merges the segment that worker w's
// range starts inside, when w is the first worker starting inside it (every cut segment
// has exactly one such worker), rows 16 y .. 16 y + 15 of its head tile: out = sum_j
// O_j 2^(m_j - M) / sum_j l_j 2^(m_j - M) over the segment's pieces j (partials in worker
// order; M the largest m_j).
constexpr int kMergeThreads = 128;
constexpr int kMergeRowsPerWarp = 4;
constexpr int kMergeRows = kMergeThreads / 32 * kMergeRowsPerWarp;  // rows per block

template <int D>
__global__ void __launch_bounds__(kMergeThreads, 6) merge_tc_kernel(const DecodeParams p) {
  __shared__ int64_t s_part[kMergeThreads / 32];
  __shared__ int s_b;
  __shared__ int64_t s_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.num_seqs;
  const int segs = p.num_kv_heads * p.n_ht;
  const int cap = p.max_blocks * p.page_size;
  const int hps = p.heads_per_seg;

  // The work list as the decode split it (seq_lens is not written by the decode).
  int64_t mine = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x)
    mine += static_cast<int64_t>((tc_eff_len(__ldg(p.seq_lens + b), cap) + kTcBlk - 1) / kTcBlk) * segs;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if (lane == 0) s_part[warp] = mine;
  if (threadIdx.x == 0) s_b = -1;
  __syncthreads();
  int64_t T = 0;
  for (int i = 0; i < kMergeThreads / 32; ++i) T += s_part[i];
  const int64_t W = min(static_cast<int64_t>(p.num_workers), T);
  const int64_t w = static_cast<int64_t>(blockIdx.x) + 1;
  if (w >= W) return;
  const int64_t x = tc_wstart(w, T, W);
  __syncthreads();
  {
    int64_t base = 0;
    for (int t0 = 0; t0 < B && base <= x; t0 += blockDim.x) {
      const int b = t0 + threadIdx.x;
      int64_t n = 0;
      if (b < B) n = static_cast<int64_t>((tc_eff_len(__ldg(p.seq_lens + b), cap) + kTcBlk - 1) / kTcBlk) * segs;
      int64_t incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (lane == 31) s_part[warp] = incl;
      __syncthreads();
      int64_t pre = 0, tot = 0;
      for (int i = 0; i < kMergeThreads / 32; ++i) {
        if (i < warp) pre += s_part[i];
        tot += s_part[i];
      }
      incl += pre;
      if (n > 0 && x >= base + incl - n && x < base + incl) {
        s_b = b;
        s_base = base + incl - n;
      }
      base += tot;
      __syncthreads();
    }
  }
  const int b = s_b;
  if (b < 0) return;
  const int nblk = (tc_eff_len(__ldg(p.seq_lens + b), cap) + kTcBlk - 1) / kTcBlk;
  const int seg = static_cast<int>((x - s_base) / nblk);
  const int64_t seg_base = s_base + static_cast<int64_t>(seg) * nblk;
  if (seg_base == x) return;  // worker w starts at a segment start: nothing is cut there
  const int64_t wf = tc_worker_of(seg_base, T, W);
  if (wf + 1 != w) return;    // a worker before w also starts inside this segment
  const int64_t wl = tc_worker_of(seg_base + nblk - 1, T, W);
  const int np = static_cast<int>(wl - wf + 1);
  // Piece j belongs to worker wf + j: for j > 0 it is that worker's first piece (slot 0);
  // worker wf's piece is its first only if its range starts at the segment start.
  const int64_t slot0 = wf * 2 + (seg_base == tc_wstart(wf, T, W) ? 0 : 1);
  auto slot_of = [&](int j) -> int64_t { return j == 0 ? slot0 : (wf + j) * 2; };
  const int kvh = seg / p.n_ht, ht = seg % p.n_ht;
  const int nrows = min(hps, p.group * p.q_len - ht * hps);
  const int64_t row0 = static_cast<int64_t>(b) * p.num_heads + kvh * p.group + ht * hps;
  // Memory row of segment row h (several query tokens: row h is token h / group's head
  // h % group; one segment per kv head then).
  auto out_row = [&](int h) -> int64_t {
    return p.q_len > 1
               ? (static_cast<int64_t>(b) * p.q_len + h / p.group) * p.num_heads + kvh * p.group + h % p.group
               : row0 + h;
  };
  const int h0 = blockIdx.y * kMergeRows + warp * kMergeRowsPerWarp;
  if (h0 >= nrows) return;

  ptx::pdl_wait_prerequisites();  // the partials are the decode's
  // Per row: M = max_j m_j and L = sum_j l_j 2^(m_j - M) with lanes across pieces (lane j
  // keeps piece j's (m, l) when there are at most 32), then out = sum_j 2^(m_j - M) O_j / L
  // with lanes across columns, the O loads of the first pieces issued with the (m, l) loads.
  constexpr int CW = D / 32;  // columns per lane
  using VecT = typename std::conditional<CW == 4, float4, float2>::type;
  auto o_ptr = [&](int j, int h) -> const VecT* {
    return reinterpret_cast<const VecT*>(p.part_o + (slot_of(j) * hps + h) * D) + lane;
  };
  for (int r = 0; r < kMergeRowsPerWarp; ++r) {
    const int h = h0 + r;
    if (h >= nrows) break;
    float2 mlj = make_float2(-INFINITY, 0.f);  // lane j: piece j's (max, sum)
    if (lane < np) mlj = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (slot_of(lane) * hps + h) * 2));
    VecT o4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o4[j] = j < np ? __ldcg(o_ptr(j, h)) : VecT{};
    float M = mlj.x;
    for (int j = lane + 32; j < np; j += 32)
      M = fmaxf(M, __ldcg(p.part_ml + (slot_of(j) * hps + h) * 2));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float Lp = mlj.y * ptx::ex2(mlj.x - Mu);
    for (int j = lane + 32; j < np; j += 32) {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (slot_of(j) * hps + h) * 2));
      Lp += t.y * ptx::ex2(t.x - Mu);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, off);
    const float iv = Lp > 0.f ? 1.f / Lp : 0.f;
    const float wl = ptx::ex2(mlj.x - Mu) * iv;  // lane j: piece j's weight (j < 32)
    auto weight = [&](int j) -> float {
      if (j < 32) return __shfl_sync(0xffffffffu, wl, j);
      return ptx::ex2(__ldcg(p.part_ml + (slot_of(j) * hps + h) * 2) - Mu) * iv;
    };
    float acc[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) acc[c] = 0.f;
    auto add = [&](float wj, const VecT& v) {
      if constexpr (CW == 4) {
        acc[0] = fmaf(wj, v.x, acc[0]); acc[1] = fmaf(wj, v.y, acc[1]);
        acc[2] = fmaf(wj, v.z, acc[2]); acc[3] = fmaf(wj, v.w, acc[3]);
      } else {
        acc[0] = fmaf(wj, v.x, acc[0]); acc[1] = fmaf(wj, v.y, acc[1]);
      }
    };
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float wj = weight(j < np ? j : 0);
      if (j < np) add(wj, o4[j]);
    }
    for (int j0 = 4; j0 < np; j0 += 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) o4[j] = j0 + j < np ? __ldcg(o_ptr(j0 + j, h)) : VecT{};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float wj = weight(j0 + j < np ? j0 + j : 0);
        if (j0 + j < np) add(wj, o4[j]);
      }
    }
    uint16_t* dst = p.out + out_row(h) * D + lane * CW;
    if constexpr (CW == 4) {
      uint2 o;
      o.x = ptx::pack_bf16x2(acc[0], acc[1]);
      o.y = ptx::pack_bf16x2(acc[2], acc[3]);
      *reinterpret_cast<uint2*>(dst) = o;
    } else {
      *reinterpret_cast<uint32_t*>(dst) = ptx::pack_bf16x2(acc[0], acc[1]);
    }
  }
}

// ------------------------------------------------------------------ host side
namespace {
template <int D, bool F8 = false>
constexpr size_t tc_smem_bytes() {
  using GE = TcGeo<D, F8>;
  return 1024 + static_cast<size_t>(GE::kStages) * GE::kStage + static_cast<size_t>(GE::kRawStages) * GE::kRawStage +
         GE::kQTile + (GE::kStages + GE::kRawStages) * sizeof(TcStageInfo) + 16 * GE::kStages +
         16 * GE::kRawStages + 24 * kTcBufs + 64 + 128 + kTcSoftThreads / 32 * kStgFloats * sizeof(float);
}
static_assert(tc_smem_bytes<128, true>() <= 227 * 1024 && tc_smem_bytes<64, true>() <= 227 * 1024 &&
                  tc_smem_bytes<128>() <= 227 * 1024 && tc_smem_bytes<64>() <= 227 * 1024,
              "shared memory per CTA");

template <int D, bool MQ, bool F8 = false>
cudaError_t launch_tc_t(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tq, int grid, cudaStream_t stream, bool overlap) {
  auto kern = decode_tc_kernel<D, MQ, F8>;
  constexpr size_t smem = tc_smem_bytes<D, F8>();
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
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, p);
  if (e != cudaSuccess || grid < 2) return e;
  // The split merge: one block column per worker boundary, launched so that it can be
  // resident while the decode drains (it waits for the decode's completion itself).
  cudaLaunchConfig_t mc = {};
  mc.gridDim = dim3(grid - 1, (p.heads_per_seg + kMergeRows - 1) / kMergeRows);
  mc.blockDim = dim3(kMergeThreads);
  mc.stream = stream;
  mc.attrs = attr;
  mc.numAttrs = 1;
  return cudaLaunchKernelEx(&mc, merge_tc_kernel<D>, p);
}
}  // namespace

size_t decode_tc_smem_bytes(int head_dim, bool fp8) {
  if (fp8) return head_dim == 64 ? tc_smem_bytes<64, true>() : tc_smem_bytes<128, true>();
  return head_dim == 64 ? tc_smem_bytes<64>() : tc_smem_bytes<128>();
}

cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tq, int grid, cudaStream_t stream, bool overlap) {
  if (p.k_scales != nullptr)
    return p.head_dim == 64 ? launch_tc_t<64, false, true>(p, tk, tv, tq, grid, stream, overlap)
                            : launch_tc_t<128, false, true>(p, tk, tv, tq, grid, stream, overlap);
  if (p.q_len > 1)
    return p.head_dim == 64 ? launch_tc_t<64, true>(p, tk, tv, tq, grid, stream, overlap)
                            : launch_tc_t<128, true>(p, tk, tv, tq, grid, stream, overlap);
  if (p.head_dim == 64) return launch_tc_t<64, false>(p, tk, tv, tq, grid, stream, overlap);
  return launch_tc_t<128, false>(p, tk, tv, tq, grid, stream, overlap);
}

}  // namespace gqa
