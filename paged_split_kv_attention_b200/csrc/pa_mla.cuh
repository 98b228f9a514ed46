// pa_mla.cuh -- MLA (shared-latent) paged split-KV decode: the partition pass on
// the 5th-generation tensor cores, run by pairs of SMs (2-SM tcgen05 MMAs).
//
// What it computes.  All H = 128 query heads of a sequence read one compressed
// latent vector per token (page "wenku.it search: Multi-head Latent Attention
// (MLA)", DeepSeek-V2 abstract on the latent KV): the key is the whole
// 576-wide latent row and the value its first 512 dims, so per sequence
//   out[h, :] = softmax_t(scale * q[h, :] . c_t) c_t[0:512].
// The KV stream is split and merged exactly as for GQA (page
// "cidian.kuaisou.com: flash decoding ++", three-step snippets): the flattened
// stream of 128-token tiles is cut into equal pieces, one per CTA pair; a piece
// that covers a whole sequence writes the output, otherwise it leaves a
// normalised partial and the log-sum-exp of each head row for the merge kernel.
//
// Why a pair of SMs, and how the work is split.  The value accumulator of a
// sequence (128 heads x 512 fp32) is as large as one SM's whole tensor memory,
// so a piece runs on a cluster of two CTAs (on two SMs) and every MMA is a 2-SM
// MMA (cta_group::2) issued by the rank-0 CTA: each CTA supplies half of the A
// rows and half of the B rows, and each CTA's tensor memory receives its half of
// the result rows.
//   - Heads: CTA r owns heads [64r, 64r+64) (the A rows: the query for the score
//     MMA, P for the value MMA).
//   - Scores: S = Q C^T, M = 128 heads, N = 128 tokens, K = 576.  CTA r stages
//     its own 64 tokens of the tile (all 576 dims, 72 KB) as its half of B.  The
//     scores are computed once for the pair, at N = 128.
//   - Values: O += P V, M = 128 heads, N = 256 dims per MMA, two MMAs for the
//     512 dims, K = the tile's 128 tokens.  Each CTA supplies 128 of every 256
//     dims (B is split by N), for all 128 tokens: its own tokens are staged
//     already, and the other CTA's tokens are fetched for the CTA's value dims
//     only (32 KB, an L2 hit: the other CTA has just loaded them from HBM)
//     into the slabs of the stage that only the score MMA needed.
// So the latent is read from HBM once, the scores are not recomputed, and each
// SM stages 72 KB per 128 tokens.
//
// Tensor memory per CTA (512 columns, "2x2" layout of a 2-SM M=128 result: lane
// l < 64 holds head l with the first half of the columns, lane 64 + l the same
// head with the second half):
//   [0, 128)    two score buffers of 64 columns (64 heads x 128 tokens)
//   [128, 256)  query dims [0, 256) as the A operand of the score MMA (each head's
//               row present in lanes l and 64 + l)
//   [256, 512)  value accumulator: 64 heads x 512 dims
// Shared memory per CTA: two 72 KB latent stages, query dims [256, 576) (40 KB),
// P as a bf16 hi + lo pair (2 x 16 KB, the A operand of the value MMA).
//
// Warp roles (192 threads per CTA).  Warps 0-3 (thread t: head 64r + t % 64,
// token half t / 64 of each tile): query loads, the online softmax in log2 units
// (each head's two threads agree on the running max through shared memory, with
// a lazily raised max), P as bf16 hi + lo (about 16 significant bits: a single
// bf16 copy biases the value mix by up to 2^-9 per weight), zeroing value rows
// past a ragged end, and the epilogue.  Warp 4 issues the TMA loads: its own
// tokens (completion counted on the rank-0 CTA's barrier, so that the MMA issuer
// sees both halves land), and, once the tile's scores are done, the other CTA's
// tokens for its value dims.  Warp 5 of the rank-0 CTA issues every MMA from one
// thread.  Every wait is bounded.
#pragma once

#include "pa_device.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kMlaTile = 128;             // tokens per tile (the pair's)
constexpr int kMlaHalf = 64;              // tokens of a tile staged by each CTA
constexpr int kMlaBox = 32;               // rows per TMA box (block sizes: multiples of 32)
constexpr int kMlaHeads = 128;
constexpr int kMlaDk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaStages = 2;
constexpr int kMlaThreads = 192;
constexpr int kMlaRescale = 8;            // raise the running max only past 2^8 growth

struct MlaParams {
  const uint16_t *q;            // [B][128][576]
  const int32_t *block_table;   // [B][mbs]
  const int32_t *context_lens;  // [B]
  void *out;                    // [B][128][512] bf16
  float *part_o;                // [slots][128][512]
  float *part_lse;              // [slots][128], log2 units
  int B, bs, mbs, nb;
  int parts;                    // pieces (CTA pairs)
  int min_tiles;                // > 0: at least this many tiles per piece (automatic launches)
  float scale_log2;
  int wide;                     // block size a multiple of 64: a CTA's 64 tokens of a tile lie
                                // in one block and move as whole-slab 3-D boxes
};

struct MlaLayout {
  static constexpr int kSlab = kMlaHalf * 128;            // 64 rows x 64 bf16 = 8 KB
  static constexpr int kSlabs = kMlaDk / 64;              // 9 slabs per staged half tile
  static constexpr int kStage = kSlabs * kSlab;           // 72 KB
  static constexpr int kQSlabs = 5;                       // query dims [256, 576)
  static constexpr int stage = 0;
  static constexpr int qs = stage + kMlaStages * kStage;
  // P pool: slabs 0, 1 = P hi of token half 1 for tiles of even / odd index, 2, 3 =
  // P lo of token halves 0, 1; P hi of token half 0 goes into slab 8 of the tile's
  // own stage (the rope dims, free once the tile's scores are done)
  static constexpr int ps = qs + kQSlabs * kSlab;
  static constexpr int bars = ps + 4 * kSlab;
  static constexpr int nbars = 17;
  static constexpr int xch = bars + nbars * 8;            // float xm[2][128], xl[128]
  static constexpr int misc = xch + 3 * 128 * 4;         // tmem base, abort, scan, start
  static constexpr int end = misc + 128;
  static constexpr size_t bytes() { return 1024 + end; }
  static_assert(kStage % 1024 == 0 && qs % 1024 == 0 && ps % 1024 == 0,
                "swizzled tiles need 1 KB alignment");
};
static_assert(MlaLayout::bytes() <= 232448, "shared memory per CTA");

// Tensor memory columns (exactly 512, allocated for the pair)
constexpr int kTmS = 0;        // score buffers at 0, 64
constexpr int kTmQ = 128;      // query dims [0, 256): 16 k-steps x 8 columns
constexpr int kQTmemDims = 256;
constexpr int kTmO = 256;      // value accumulator: dims block 0 at 256, block 1 at 384

// tiles of 128 tokens in a sequence of c tokens (c clamped to [0, cap])
__device__ __forceinline__ int mla_tiles(int c, int cap) {
  return (min(max(c, 0), cap) + kMlaTile - 1) / kMlaTile;
}

// Walks the tiles of a piece in order: sequence b, tile j within it, its tile
// count P, and whether the tile opens / closes that sequence's run in the piece.
struct MlaCursor {
  const int32_t *cl;
  int B, cap, n, ntiles, b, j, P, ctx;
  __device__ void init(const MlaParams &p, int b0, int j0, int nt) {
    cl = p.context_lens;
    B = p.B;
    cap = p.mbs * p.bs;
    n = 0;
    ntiles = nt;
    b = b0;
    j = j0;
    ctx = b < B ? min(max(__ldg(&cl[b]), 0), cap) : 0;
    P = (ctx + kMlaTile - 1) / kMlaTile;
  }
  __device__ bool first() const { return n == 0 || j == 0; }
  __device__ bool last() const { return n == ntiles - 1 || j == P - 1; }
  __device__ void next() {
    ++n;
    if (++j >= P) {
      j = 0;
      P = 0;
      while (P == 0 && b < B - 1) {                  // skip empty sequences
        ctx = min(max(__ldg(&cl[++b]), 0), cap);
        P = (ctx + kMlaTile - 1) / kMlaTile;
      }
    }
  }
};

// Cache row of the 32-token box k (0..3) of tile j of sequence b: -1 for a block
// id out of range, -2 for a box that lies wholly past the context (not loaded).
__device__ __forceinline__ int mla_box_row(const MlaParams &p, int b, int j, int k, int ctx) {
  const int t = j * kMlaTile + k * kMlaBox;
  if (t >= ctx) return -2;
  const int blk = __ldg(&p.block_table[static_cast<long long>(b) * p.mbs + t / p.bs]);
  if (blk < 0 || blk >= p.nb) return -1;
  return blk * p.bs + t % p.bs;
}

// Tokens of the tile's half `half` (0: the rank-0 CTA's 64, 1: the other's) that
// lie inside a context of ctx tokens.
__device__ __forceinline__ int mla_half_tokens(int ctx, int j, int half) {
  return min(max(ctx - j * kMlaTile - half * kMlaHalf, 0), kMlaHalf);
}

// barrier slots.  Local: each CTA waits on its own.  Pair: live in the rank-0
// CTA only (arrivals from both CTAs); the same slots are unused in the other.
enum MlaBar {
  kLatEmpty = 0,    // [2] local: the value MMA of the stage's tile is done (commit to both)
  kSFull = 2,       // [2] local: scores of tile n in buffer n%2 (commit to both)
  kOReady = 4,      // [2] local: value MMA of tile n done (commit to both; one slot per
                    //     parity so that a waiter is never two phases behind)
  kPvFull = 6,      // [2] local: the other CTA's tokens landed in this CTA's value slabs
  kQEmpty = 8,      // local: last score MMA of a sequence done (commit to both)
  kFinal = 9,       // local: every MMA done (commit to both)
  kStall = 10,      // local, test hook only: nothing ever arrives here
  kLatFull = 11,    // [2] pair: both CTAs' own tokens landed (2 arrivals + bytes)
  kPhiFull = 13,    // pair: P hi of the tile written, its value rows in place (8 warps)
  kQFull = 14,      // pair: query of a sequence in place in both CTAs (8 warps + 2 copies)
  kOFree = 15,      // pair: both epilogues have read the accumulator (8 warps)
  kPloFull = 16     // pair: P lo of the tile written in both CTAs (8 warps)
};

__global__ void __launch_bounds__(kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_q, const MlaParams p) {
  using L = MlaLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::bars);
  float *xm = reinterpret_cast<float *>(sm + L::xch);            // [2][128] row maxima
  float *xl = xm + 2 * 128;                                        // [128] row sums
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(sm + L::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::misc + 4);
  int *scan_scratch = reinterpret_cast<int *>(sm + L::misc + 16);   // [6]
  int *start = reinterpret_cast<int *>(sm + L::misc + 48);          // b, j of the first tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = pair::rank();        // 0: issues the MMAs; heads [64 rank, +64)
  const int pc = blockIdx.x >> 1;            // which piece of the tile stream
  const int cap = p.mbs * p.bs;

  // ---- prologue (all threads): tiles per sequence, block-wide scan, the piece
  // [tb, te) of the flattened tile stream and the (sequence, tile) it starts at
  long long tb, te;
  {
    const int per = (p.B + kMlaThreads - 1) / kMlaThreads;
    const int b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) {
      const int c = __ldg(&p.context_lens[b]);
      if (blockIdx.x == 0 && (c < 0 || c > cap)) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
      local += mla_tiles(c, cap);
    }
    int v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += x;
    }
    if (lane == 31) scan_scratch[warp] = v;
    if (tid == 0) {
      start[0] = 0;
      start[1] = 0;
    }
    __syncthreads();
    int run = v - local, total = 0;
    for (int i = 0; i < kMlaThreads / 32; ++i) {
      if (i < warp) run += scan_scratch[i];
      total += scan_scratch[i];
    }
    const long long TP = total;
    const int pieces = used_pieces(p.parts, TP, p.min_tiles, p.B);
    tb = pc < pieces ? piece_begin(pc, TP, pieces) : 0;
    te = pc < pieces ? piece_begin(pc + 1, TP, pieces) : 0;
    for (int b = b0; b < b1; ++b) {
      const int P = mla_tiles(__ldg(&p.context_lens[b]), cap);
      if (P > 0 && run <= tb && tb < run + P) {
        start[0] = b;
        start[1] = static_cast<int>(tb - run);
      }
      run += P;
    }
  }
  if (tid == 0) {
    for (int i = 0; i < L::nbars; ++i) {
      uint32_t cnt = 1;
      if (i == kLatFull || i == kLatFull + 1) cnt = 2;
      if (i == kPhiFull || i == kPloFull || i == kOFree) cnt = 8;
      if (i == kQFull) cnt = 10;          // 8 warps + each CTA's query copy (with its bytes)
      mbar_init(&bar[i], cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_base_s))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync();            // both CTAs' barriers are initialised before any remote use
  tc_fence_after();

  const uint32_t tmem = *tmem_base_s;
  // empty sequences: all-zero rows (the rank-0 CTA of each piece takes a share)
  if (rank == 0)
    for (int b = pc; b < p.B; b += p.parts)
      if (mla_tiles(__ldg(&p.context_lens[b]), cap) == 0)
        for (int i = tid; i < kMlaHeads * kMlaDv; i += kMlaThreads)
          reinterpret_cast<uint16_t *>(p.out)[static_cast<long long>(b) * kMlaHeads * kMlaDv + i] = 0;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int ntiles = static_cast<int>(te - tb);
  const int b_first = start[0], j_first = start[1];
  // the pair barriers, addressed in the rank-0 CTA
  const uint32_t phifull_pair = pair::map_to(&bar[kPhiFull], 0);
  const uint32_t plofull_pair = pair::map_to(&bar[kPloFull], 0);
  const uint32_t qfull_pair = pair::map_to(&bar[kQFull], 0);
  const uint32_t ofree_pair = pair::map_to(&bar[kOFree], 0);
  // this CTA's value dims: latent slabs {2r, 2r+1, 4+2r, 5+2r}; the other CTA's
  // tokens for them are staged in the slabs of the same index xor 2
  const int vs0 = 2 * static_cast<int>(rank);

  if (warp == 4) {
    // ------------------------------------------------------------ copy issue
    // Lane i holds the cache rows of the four 32-token boxes of tile wb + i
    // (current window) and wb + 32 + i (next window); lane 0 issues, whichever of
    // "own tokens of tile n" (stage free) and "other tokens of tile n" (scores of
    // tile n done) is ready first.
    const uint64_t pol_keep = l2_evict_last_policy();
    const uint64_t pol_once = l2_evict_first_policy();
    bool aborted = false;
    if (blockIdx.x == 0 && stall_test_enabled()) {
      // Test hook for the timeout path: wait, before anything is issued, on a
      // barrier that nothing completes.  The bounded wait gives up after about a
      // second, records PA_ERR_TIMEOUT and raises the CTA's abort flag; every
      // other wait of the pair then runs out too, no copy or MMA is in flight,
      // and tensor memory is released as usual.
      const bool got = lane != 0 || mbar_wait_idle(&bar[kStall], 0, abort_flag);
      aborted = !__all_sync(0xffffffffu, got);
    }
    if (lane == 0) {
      prefetch_tensormap(&tm_a);
      if (p.wide) prefetch_tensormap(&tm_b);
    }
    MlaCursor cur;
    cur.init(p, b_first, j_first, ntiles);
    // Cache rows of the tile's boxes held by this lane: this CTA's two (own) and
    // the other CTA's two (oth), for the current window (c*) and the next (n*)
    const int own_box = 2 * static_cast<int>(rank), oth_box = 2 - own_box;
    int c_own0 = -2, c_own1 = -2, c_oth0 = -2, c_oth1 = -2;
    int n_own0 = -2, n_own1 = -2, n_oth0 = -2, n_oth1 = -2;
    auto look_up = [&](int base, int &o0, int &o1, int &t0, int &t1) {
      const int n = min(32, ntiles - base);
      int mb = 0, mj = 0, mctx = 0;
      for (int i = 0; i < n; ++i, cur.next())
        if (lane == i) {
          mb = cur.b;
          mj = cur.j;
          mctx = cur.ctx;
        }
      const bool ok = lane < n;
      o0 = ok ? mla_box_row(p, mb, mj, own_box, mctx) : -2;
      o1 = ok ? mla_box_row(p, mb, mj, own_box + 1, mctx) : -2;
      t0 = ok ? mla_box_row(p, mb, mj, oth_box, mctx) : -2;
      t1 = ok ? mla_box_row(p, mb, mj, oth_box + 1, mctx) : -2;
    };
    int wb = 0;                      // first tile of the current window
    if (ntiles > 0) look_up(0, c_own0, c_own1, c_oth0, c_oth1);
    if (ntiles > 32) look_up(32, n_own0, n_own1, n_oth0, n_oth1);
    // rows of tile n (all lanes call): k = 0, 1 own boxes, 2, 3 the other CTA's
    auto row_of = [&](int n, int k) {
      const bool w = n - wb >= 32;
      const int v = k == 0 ? (w ? n_own0 : c_own0) : k == 1 ? (w ? n_own1 : c_own1)
                  : k == 2 ? (w ? n_oth0 : c_oth0) : (w ? n_oth1 : c_oth1);
      return __shfl_sync(0xffffffffu, v, (n - wb) & 31);
    };
    int n_own = 0, n_pv = 0;
    uint64_t t_idle = globaltimer();
    uint32_t spins = 0;
    while (n_pv < ntiles && !aborted) {
      // slide the windows once the other-token loads have left the current one
      if (n_pv >= wb + 32) {
        c_own0 = n_own0;
        c_own1 = n_own1;
        c_oth0 = n_oth0;
        c_oth1 = n_oth1;
        wb += 32;
        if (ntiles > wb + 32) look_up(wb + 32, n_own0, n_own1, n_oth0, n_oth1);
      }
      int act = 0;
      if (lane == 0) {
        if (n_own < ntiles && n_own < n_pv + kMlaStages &&
            (n_own < kMlaStages ||
             mbar_test(&bar[kLatEmpty + n_own % kMlaStages], ((n_own / kMlaStages) & 1) ^ 1)))
          act = 1;
        else if (n_pv < n_own &&
                 mbar_test(&bar[kSFull + n_pv % kMlaStages], (n_pv / kMlaStages) & 1))
          act = 2;
      }
      act = __shfl_sync(0xffffffffu, act, 0);
      if (act == 1) {
        const int n = n_own++;
        const int st = n % kMlaStages;
        const int r0 = row_of(n, 0), r1 = row_of(n, 1);
        // the own tokens of the tile that next uses this stage, pulled into L2 now
        // (one copy instruction): their load, issued once this tile's value MMA is
        // done, then finds them in L2
        const int f0 = p.wide && n + kMlaStages < ntiles ? row_of(n + kMlaStages, 0) : -2;
        if (lane == 0) {
          if (f0 >= 0) tma_prefetch_3d(&tm_a, 0, f0, 0, pol_keep);
          if (r0 == -1 || r1 == -1) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
          const uint32_t bytes =
              p.wide ? (r0 >= 0 ? L::kStage : 0)
                     : L::kSlabs * kMlaBox * 128 * ((r0 >= 0) + (r1 >= 0));
          const uint32_t full = pair::map_to(&bar[kLatFull + st], 0);
          pair::arrive_expect_tx_remote(full, bytes);
          uint8_t *dst = sm + L::stage + st * L::kStage;
          if (p.wide) {
            // the 64 tokens in one copy: a 64 dims x 64 rows x 9 slabs box lands as
            // the stage's 9 slabs (r1 is r0's second half, or past the context)
            if (r0 >= 0) pair::tma_load_3d_to_pair_bar(dst, &tm_a, full, 0, r0, 0, pol_keep);
          } else {
#pragma unroll 1
            for (int s = 0; s < L::kSlabs; ++s) {
              if (r0 >= 0)
                pair::tma_load_2d_to_pair_bar(dst + s * L::kSlab, &tm_a, full, 64 * s, r0,
                                              pol_keep);
              if (r1 >= 0)
                pair::tma_load_2d_to_pair_bar(dst + s * L::kSlab + kMlaBox * 128, &tm_a, full,
                                              64 * s, r1, pol_keep);
            }
          }
        }
      } else if (act == 2) {
        const int n = n_pv++;
        const int st = n % kMlaStages;
        const int r0 = row_of(n, 2), r1 = row_of(n, 3);
        if (lane == 0) {
          const uint32_t bytes = p.wide ? (r0 >= 0 ? 4 * L::kSlab : 0)
                                        : 4 * kMlaBox * 128 * ((r0 >= 0) + (r1 >= 0));
          mbar_arrive_expect_tx(&bar[kPvFull + st], bytes);
          // the value dims: latent slabs vs0, vs0 + 1, vs0 + 4, vs0 + 5, into the
          // stage's slabs of index xor 2
          uint8_t *dst = sm + L::stage + st * L::kStage;
          if (p.wide) {
            // two 64 dims x 64 rows x 2 slabs boxes
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int sl = vs0 + 4 * g;
              if (r0 >= 0)
                tma_load_3d_hint(dst + (sl ^ 2) * L::kSlab, &tm_b, &bar[kPvFull + st], 0, r0, sl,
                                 pol_once);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int sl = vs0 + (i & 1) + 4 * (i >> 1);
              if (r0 >= 0)
                tma_load_2d_hint(dst + (sl ^ 2) * L::kSlab, &tm_a, &bar[kPvFull + st], 64 * sl, r0,
                                 pol_once);
              if (r1 >= 0)
                tma_load_2d_hint(dst + (sl ^ 2) * L::kSlab + kMlaBox * 128, &tm_a,
                                 &bar[kPvFull + st], 64 * sl, r1, pol_once);
            }
          }
        }
      }
      if (act != 0) {
        spins = 0;
      } else if ((++spins & 63u) == 0) {
        if (spins == 64) t_idle = globaltimer();
        bool stop = false;
        if (lane == 0) {
          if (*abort_flag) stop = true;
          else if (globaltimer() - t_idle > PA_WAIT_TIMEOUT_NS) {
            record_error(5 /* PA_ERR_TIMEOUT */);
            *abort_flag = 1;
            stop = true;
          }
        }
        aborted = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      }
    }
    if (lane == 0 && aborted) {
      // leave no copy in flight into this CTA's shared memory: the other-token
      // loads complete on a local barrier (bounded wait); the own-token loads
      // count on the rank-0 CTA's barrier, so give them time to land
      volatile int never = 0;
      for (int n = n_pv > kMlaStages ? n_pv - kMlaStages : 0; n < n_pv; ++n)
        mbar_wait(&bar[kPvFull + n % kMlaStages], (n / kMlaStages) & 1, &never);
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 50000) __nanosleep(1000);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (rank == 0 && lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kMlaTile, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, 256, true);
      // descriptors are a base descriptor plus the byte offset / 16 (address field
      // in the low bits); every offset added below is a compile-time constant
      const uint64_t b_desc0 = umma_desc(smem_u32(sm + L::stage), 16, 1024);        // K-major
      const uint64_t v_desc0 = umma_desc(smem_u32(sm + L::stage), L::kSlab, 1024);  // MN-major
      const uint64_t q_desc0 = umma_desc(smem_u32(sm + L::qs), 16, 1024);
      const uint64_t p_desc0 = umma_desc(smem_u32(sm + L::ps), 16, 1024);
      const uint64_t pst_desc0 = umma_desc(smem_u32(sm + L::stage), 16, 1024);  // K-major P
      int s_seg = -1, o_seg = -1;
      MlaCursor cs, cp;                  // tile walks of the score and value MMAs
      cs.init(p, b_first, j_first, ntiles);
      cp.init(p, b_first, j_first, ntiles);
      auto issue_s = [&](int n) {
        const int st = n % kMlaStages;
        const bool first = cs.first();
        const bool last = cs.last();
        cs.next();
        if (first) ++s_seg;
        tc_fence_after();
        const uint64_t bst = b_desc0 + ((st * L::kStage) >> 4);
        const uint32_t d = tmem + kTmS + (n % 2) * (kMlaTile / 2);
        // 16-dim step ks reads latent slab ks/4 at byte offset 32 (ks%4) of each row
#pragma unroll
        for (int ks = 0; ks < kMlaDk / 16; ++ks) {
          const uint64_t b = bst + (((ks >> 2) * L::kSlab + (ks & 3) * 32) >> 4);
          if (ks < kQTmemDims / 16) {
            pair::mma_ts(d, tmem + kTmQ + ks * 8, b, idesc_s, ks > 0);
          } else {
            const int kq = ks - kQTmemDims / 16;
            pair::mma_ss(d, q_desc0 + (((kq >> 2) * L::kSlab + (kq & 3) * 32) >> 4), b, idesc_s,
                         true);
          }
        }
        pair::commit_both(&bar[kSFull + n % 2]);
        if (last) pair::commit_both(&bar[kQEmpty]);
      };
      // The value MMA of tile n in two passes: P hi (written as soon as the softmax
      // is done), then P lo (whose single buffer the previous tile's lo pass must
      // have released).  Dims block nb: the CTAs supply dims [256nb, 256nb+128)
      // and [256nb+128, 256nb+256); token half h of the tile sits in slabs
      // 4nb + 2h, 4nb + 2h + 1 of both CTAs (own tokens or the other CTA's, see
      // above); 16 tokens (2 KB) per step.
      auto issue_pv = [&](int n, bool lo_pass) {
        const int st = n % kMlaStages;
        bool first = false;
        if (!lo_pass) {
          first = cp.first();
          cp.next();
          if (first) ++o_seg;
        }
        tc_fence_after();
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t vb = v_desc0 + ((st * L::kStage + (4 * nb + 2 * h) * L::kSlab) >> 4);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              uint64_t a;
              if (lo_pass)
                a = p_desc0 + (((2 + h) * L::kSlab + kq * 32) >> 4);
              else if (h == 0)
                a = pst_desc0 + ((st * L::kStage + 8 * L::kSlab + kq * 32) >> 4);
              else
                a = p_desc0 + (((n & 1) * L::kSlab + kq * 32) >> 4);
              const uint64_t b = vb + ((kq * 2048) >> 4);
              pair::mma_ss(tmem + kTmO + nb * 128, a, b, idesc_o,
                           lo_pass || !(first && h == 0 && kq == 0));
            }
          }
        }
        if (lo_pass) {
          pair::commit_both(&bar[kLatEmpty + st]);
          pair::commit_both(&bar[kOReady + n % 2]);
        }
      };
      // S(m), PVhi(m) and PVlo(m) are each issued in tile order, whichever is ready
      // first: S(m) once PVhi(m-2) is issued (it reuses that score buffer, which
      // the softmax had read before writing P hi; the tensor pipe runs one
      // thread's MMAs in order), both CTAs' own tokens of tile m have landed and,
      // at a sequence start, the query is in place; PVhi(m) once P hi is written
      // and the value rows are in place in both CTAs and, at a sequence start, the
      // previous O has been read out; PVlo(m) once P lo is written.
      int ns = 0, nh = 0, nl = 0;
      uint64_t t_idle = globaltimer();
      uint32_t spins = 0;
      while (nl < ntiles) {
        bool did = false;
        if (ns < ntiles && ns < nh + 2 &&
            pair::test_cluster(&bar[kLatFull + ns % kMlaStages], (ns / kMlaStages) & 1) &&
            (!cs.first() || pair::test_cluster(&bar[kQFull], (s_seg + 1) & 1))) {
          issue_s(ns++);
          did = true;
        }
        if (nh < ns && pair::test_cluster(&bar[kPhiFull], nh & 1) &&
            (!cp.first() || o_seg < 0 || pair::test_cluster(&bar[kOFree], o_seg & 1))) {
          issue_pv(nh++, false);
          did = true;
        }
        if (nl < nh && pair::test_cluster(&bar[kPloFull], nl & 1)) {
          issue_pv(nl++, true);
          did = true;
        }
        if (did) {
          spins = 0;
        } else if ((++spins & 63u) == 0) {
          if (spins == 64) t_idle = globaltimer();
          if (*abort_flag || globaltimer() - t_idle > PA_WAIT_TIMEOUT_NS) {
            if (!*abort_flag) record_error(5 /* PA_ERR_TIMEOUT */);
            *abort_flag = 1;
            break;
          }
        }
      }
    }
    // every MMA issued has completed before tensor memory is released (an issuer
    // with nothing to do commits at once)
    if (rank == 0 && lane == 0) pair::commit_both(&bar[kFinal]);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue (warps 0-3)
    const int t = tid;                                 // TMEM lane
    const int lh = t & 63;                             // head 64 rank + lh
    const int hh = t >> 6;                             // token half of each tile
    const int head = 64 * static_cast<int>(rank) + lh;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool aborted = false;

    // Query of sequence b.  Dims [256, 576) of the CTA's 64 heads land in shared
    // memory with one copy (a 64 dims x 64 rows x 5 slabs box: the 128-byte
    // swizzled K-major layout of the A operand), counted on the rank-0 CTA's
    // query barrier.  Dims [0, 256) go into TMEM lane t as bf16 pairs (both lanes
    // of the head: the layout of a 2-SM A operand), loaded in two batches of 128
    // dims.  Called after the previous sequence's last score MMA.
    auto load_query = [&](int b) {
      if (t == 0) {
        pair::arrive_expect_tx_remote(qfull_pair, L::kQSlabs * L::kSlab);
        pair::tma_load_3d_to_pair_bar(sm + L::qs, &tm_q, qfull_pair, 0,
                                      b * kMlaHeads + 64 * static_cast<int>(rank),
                                      kQTmemDims / 64, l2_evict_first_policy());
      }
      const uint4 *src = reinterpret_cast<const uint4 *>(
          p.q + (static_cast<long long>(b) * kMlaHeads + head) * kMlaDk);
#pragma unroll 1
      for (int g = 0; g < kQTmemDims / 64; g += 2) {
        uint4 x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = __ldg(src + g * 8 + i);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[4 * i] = x[8 * k + i].x;
            v[4 * i + 1] = x[8 * k + i].y;
            v[4 * i + 2] = x[8 * k + i].z;
            v[4 * i + 3] = x[8 * k + i].w;
          }
          tmem_st32u(tmem + kTmQ + (g + k) * 32 + lane_off, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::arrive_remote(qfull_pair);
    };

    // Pull the query of sequence b into L2 a tile ahead of load_query, marked to
    // stay (the latent tiles streaming meanwhile are marked the same way): the
    // TMEM part (dims [0, 256): four 128-byte lines, two per thread of the head)
    // and the shared-memory part's box.
    const uint64_t pol_q = l2_evict_last_policy();
    auto prefetch_query = [&](int b) {
      if (b < 0 || b >= p.B) return;
      const char *row = reinterpret_cast<const char *>(
          p.q + (static_cast<long long>(b) * kMlaHeads + head) * kMlaDk);
      for (int i = hh; i < kQTmemDims * 2 / 128; i += 2)
        asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(row + i * 128));
      if (t == 0)
        tma_prefetch_3d(&tm_q, 0, b * kMlaHeads + 64 * static_cast<int>(rank), kQTmemDims / 64,
                        pol_q);
    };

    // Zero rows [from, 64) of the four slabs at slab indices first, first + 1,
    // first + 4, first + 5 of a stage (value rows of tokens past a ragged end, so
    // that 0 x stale data stays 0); the 128 threads share the work.
    auto zero_rows = [&](uint8_t *stage, int first, int from) {
      const int rows = kMlaHalf - from;
      for (int i = t; i < rows * 4 * 8; i += 128) {
        const int sl = first + (i / (rows * 8) & 1) + 4 * ((i / (rows * 8)) >> 1);
        const int r = from + (i / 8) % rows, ch = i % 8;
        *reinterpret_cast<uint4 *>(stage + sl * L::kSlab + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
      }
    };

    int q_seg = 0;                       // sequences whose query has been loaded
    MlaCursor cq, cur;                   // query look-ahead walk, softmax walk
    cq.init(p, b_first, j_first, ntiles);
    cur.init(p, b_first, j_first, ntiles);
    // called with cq at tile m: load the query if m opens a sequence, step past m
    auto query_for = [&](int m) {
      if (cq.first()) {
        if (m > 0) {
          const bool got = !aborted && mbar_wait(&bar[kQEmpty], (q_seg - 1) & 1, abort_flag);
          aborted = !__all_sync(0xffffffffu, got);
          tc_fence_after();
        }
        if (!aborted) load_query(cq.b);
        ++q_seg;
      }
      cq.next();
    };

    float m_run = -INFINITY, l_run = 0.f;
    int ctx = 0;
    if (ntiles > 0) {
      prefetch_query(b_first);
      query_for(0);
    }
    for (int n = 0; n < ntiles; ++n, cur.next()) {
      const int b = cur.b, j = cur.j, P = cur.P;
      const bool first = cur.first();
      const bool last = cur.last();
      // cq is at tile n + 1: if it opens a sequence, its query is loaded at the end
      // of this iteration; pull it into L2 now
      if (n + 1 < ntiles && cq.first()) prefetch_query(cq.b);
      if (first) {
        m_run = -INFINITY;
        l_run = 0.f;
        ctx = cur.ctx;
      }
      const int st = n % kMlaStages;
      uint8_t *stage = sm + L::stage + st * L::kStage;
      const int ntok = mla_half_tokens(ctx, j, hh);
      float sc[kMlaHalf];
      {
        const bool got = !aborted && mbar_wait(&bar[kSFull + n % 2], (n / 2) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        const uint32_t scol = tmem + kTmS + (n % 2) * (kMlaTile / 2) + lane_off;
        float (&s0)[32] = *reinterpret_cast<float (*)[32]>(&sc[0]);
        float (&s1)[32] = *reinterpret_cast<float (*)[32]>(&sc[32]);
        tmem_ld32(scol, s0);
        tmem_ld32(scol + 32, s1);
        tmem_wait_ld();
      }
      // ---- online softmax (log2 units); the head's two threads agree on the max
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kMlaHalf; ++i) {
        sc[i] = i < ntok ? sc[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, sc[i]);
      }
      xm[(n & 1) * 128 + t] = mt;
      named_bar_sync(1 + (warp & 1), 64);      // warps w and w + 2 hold the same heads
      mt = fmaxf(mt, xm[(n & 1) * 128 + (t ^ 64)]);
      const bool raise = mt > m_run + kMlaRescale;
      bool pv_prev_done = n == 0;
      if (__any_sync(0xffffffffu, raise && !first)) {
        // O must be scaled by 2^(m_old - m_new) for the rows whose max moved: wait
        // until the previous tile's value MMA has landed, then rescale in TMEM
        const bool got = !aborted && mbar_wait(&bar[kOReady + (n - 1) % 2], ((n - 1) / 2) & 1,
                                               abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        pv_prev_done = true;
        const float alpha = (raise && !first) ? ex2_approx(m_run - mt) : 1.f;
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld32(tmem + kTmO + c + lane_off, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tmem + kTmO + c + lane_off, v);
        }
        tmem_wait_st();
        tc_fence_before();
        if (raise && !first) l_run *= alpha;
      }
      if (raise) m_run = mt;
      // ---- P = 2^(s - m) as a bf16 hi + lo pair, into this thread's row of the
      // A operand of the value MMA: heads x 128 tokens, K-major, 128-byte swizzle
      // (token half hh = slab hh; hi slabs first, lo slabs 16 KB on)
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int e = 0; e < kMlaHalf / 2; ++e) {
        const float p0 = ex2_approx(sc[2 * e] - m_run);
        const float p1 = ex2_approx(sc[2 * e + 1] - m_run);
        split2<true>(p0, p1, hi[e], lo[e]);
        l_run += p0 + p1;
      }
      {
        // P hi: token half 0 into slab 8 of the tile's stage, half 1 into the pool
        // slab of this tile's parity (both free: see the layout)
        uint8_t *prow = hh == 0 ? stage + 8 * L::kSlab + lh * 128
                                : sm + L::ps + (n & 1) * L::kSlab + lh * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(prow + ((c ^ (lh & 7)) << 4)) =
              make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
      }
      // ---- tokens past a ragged end: zero their value rows, own tokens now (the
      // scores are done with them), the other CTA's once they have landed
      const bool ragged = (j + 1) * kMlaTile > ctx;
      if (ragged) {
        const int own = mla_half_tokens(ctx, j, static_cast<int>(rank));
        if (own < kMlaHalf) zero_rows(stage, vs0, own);
      }
      {
        const bool got = !aborted && mbar_wait(&bar[kPvFull + st], (n / kMlaStages) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
      }
      if (ragged) {
        const int oth = mla_half_tokens(ctx, j, 1 - static_cast<int>(rank));
        if (oth < kMlaHalf) zero_rows(stage, vs0 ^ 2, oth);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::arrive_remote(phifull_pair);
      // P lo: its single buffer is released by the previous tile's lo pass
      if (!pv_prev_done) {
        const bool got = !aborted && mbar_wait(&bar[kOReady + (n - 1) % 2], ((n - 1) / 2) & 1,
                                               abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
      }
      {
        uint8_t *prow = sm + L::ps + (2 + hh) * L::kSlab + lh * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(prow + ((c ^ (lh & 7)) << 4)) =
              make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) pair::arrive_remote(plofull_pair);
      // the next tile's query, if it opens a sequence: loaded while the tensor
      // pipe runs this tile's value MMA (its score MMA, the last reader of the
      // current query, is done)
      if (n + 1 < ntiles) query_for(n + 1);
      // ---- sequence end: normalise and write this thread's half of the head row
      if (last) {
        const bool got = !aborted && mbar_wait(&bar[kOReady + n % 2], (n / 2) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        xl[t] = l_run;
        named_bar_sync(1 + (warp & 1), 64);
        const float l_tot = l_run + xl[t ^ 64];
        // the sequence's tiles all lie in this piece iff it starts and ends inside
        const bool whole = n - j >= 0 && n - j + P <= ntiles;
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        const long long slot = pc + b;
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld32(tmem + kTmO + c + lane_off, v);
          tmem_wait_ld();
          // column c of dims block c / 128: dims 256 (c / 128) + 128 hh + c % 128
          const int d0 = 256 * (c >> 7) + 128 * hh + (c & 127);
          if (whole) {
            uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                          (static_cast<long long>(b) * kMlaHeads + head) * kMlaDv + d0;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              uint4 w;
              w.x = pack2<true>(v[8 * q8] * inv, v[8 * q8 + 1] * inv);
              w.y = pack2<true>(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv);
              w.z = pack2<true>(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv);
              w.w = pack2<true>(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv);
              *reinterpret_cast<uint4 *>(o + 8 * q8) = w;
            }
          } else {
            float *o = p.part_o + (slot * kMlaHeads + head) * kMlaDv + d0;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4 *>(o + 4 * q4) = make_float4(
                  v[4 * q4] * inv, v[4 * q4 + 1] * inv, v[4 * q4 + 2] * inv, v[4 * q4 + 3] * inv);
          }
        }
        if (!whole && hh == 0)
          p.part_lse[slot * kMlaHeads + head] = l_tot > 0.f ? m_run + log2f(l_tot) : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pair::arrive_remote(ofree_pair);
      }
    }
  }

  // ---- teardown: every MMA of the pair has completed before either CTA frees
  // its tensor memory, and neither CTA leaves while the other may still signal it
  __syncthreads();
  if (warp == 5 && lane == 0) {
    volatile int never = 0;
    mbar_wait(&bar[kFinal], 0, &never);
  }
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace pa
