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
// stream of 96-token tiles (each non-empty sequence opening with a few empty
// units that stand for its fixed cost) is cut into equal pieces, one per CTA
// pair; a piece that covers a whole sequence writes the output, otherwise it
// leaves a normalised partial and the log-sum-exp of each head row for the merge
// kernel.
//
// Why a pair of SMs, and how the work is split.  The value accumulator of a
// sequence (128 heads x 512 fp32) is as large as one SM's whole tensor memory,
// so a piece runs on a cluster of two CTAs (on two SMs) and every MMA is a 2-SM
// MMA (cta_group::2) issued by the rank-0 CTA: each CTA supplies half of the A
// rows and half of the B rows, and each CTA's tensor memory receives its half of
// the result rows.
//   - Heads: CTA r owns heads [64r, 64r+64) (the A rows: the query for the score
//     MMA, P for the value MMA).
//   - Scores: S = Q C^T, M = 128 heads, N = 96 tokens, K = 576.  CTA r stages
//     its own 48 tokens of the tile (all 576 dims, 54 KB) as its half of B.  The
//     scores are computed once for the pair.  (A 2-SM MMA of M = 128 takes the
//     same time for every N up to 192, measured on B200, so 96 tokens cost as
//     much per instruction as 128; the smaller tile buys a third stage.)
//   - Values: O += P V, M = 128 heads, N = 256 dims per MMA, two MMAs for the
//     512 dims, K = the tile's 96 tokens.  Each CTA supplies 128 of every 256
//     dims (B is split by N), for all 96 tokens: its own tokens are staged
//     already, and the other CTA's tokens are fetched for the CTA's value dims
//     only (24 KB, an L2 hit: the other CTA has just loaded them from HBM) into
//     the slabs of the stage that only the score MMA needed.
// So the latent is read from HBM once, the scores are not recomputed, and each
// SM stages 54 KB per 96 tokens.  Three stages let the copies of two tiles run
// while the third is scored and mixed.
//
// Tensor memory per CTA (512 columns, "2x2" layout of a 2-SM M=128 result: lane
// l < 64 holds head l with the first half of the columns, lane 64 + l the same
// head with the second half):
//   [0, 96)     two score buffers of 48 columns (64 heads x 96 tokens), tile n in
//               buffer n % 2, each released as soon as the softmax warps have
//               read it, so a tile's scores are taken while the previous tile's
//               softmax runs
//   [96, 256)   query dims [0, 320) as the A operand of the score MMA (each
//               head's row present in lanes l and 64 + l)
//   [256, 512)  value accumulator: 64 heads x 512 dims
// Shared memory per CTA: three 54 KB latent stages, query dims [320, 576)
// (32 KB), and P as a bf16 hi + lo pair (24 KB, the A operand of the value MMA).
//
// Warp roles (352 threads per CTA).  Warps 0-7 (four threads per head: token
// half hh and column group cg of each tile, 24 tokens each): query loads, the
// online softmax in log2 units (a head's four threads agree on the running max
// through shared memory, with a lazily raised max), P as bf16 hi + lo (about 16
// significant bits: a single bf16 copy biases the value mix by up to 2^-9 per
// weight), zeroing value rows past a ragged end, and the epilogue (rows staged
// through the idle P pool, so that each store instruction covers 8 rows x 64
// bytes).  Warp 8 issues the TMA loads: its own tokens (completion counted on the
// rank-0 CTA's barrier, so that the MMA issuer sees both halves land), and, once
// the tile's scores are done, the other CTA's tokens for its value dims.  Warps 9
// and 10 of the rank-0 CTA issue the score and the value MMAs, one thread each; a
// tile's score MMA enters the tensor pipe after the value MMA of the tile two
// back.  Every wait is bounded.
#pragma once

#include <type_traits>

#include "pa_device.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kMlaTile = 96;              // tokens per tile (the pair's)
constexpr int kMlaHalf = 48;              // tokens of a tile staged by each CTA
constexpr int kMlaBox = 16;               // rows per TMA box (block sizes: multiples of 16)
constexpr int kMlaBoxes = kMlaHalf / kMlaBox;   // boxes per CTA half tile
constexpr int kMlaHeads = 128;
constexpr int kMlaDk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaStages = 3;
#ifndef PA_MLA_LOOKAHEAD
#define PA_MLA_LOOKAHEAD 2
#endif
constexpr int kMlaLookahead = PA_MLA_LOOKAHEAD;   // own-token tiles issued past the next fetch
#ifndef PA_MLA_PREFETCH
#define PA_MLA_PREFETCH 0
#endif
// tiles ahead whose own rows are pulled into L2 (0: none; with the value MMA ahead
// of the next score MMA in the pipe, a prefetch two tiles ahead cost 6 µs on B64)
constexpr int kMlaPrefetch = PA_MLA_PREFETCH;
constexpr int kMlaSoftmaxWarps = 8;       // warps 0-7: softmax and epilogue
constexpr int kMlaProducer = 8;           // warp 8: copy issue
constexpr int kMlaIssuer = 9;             // warp 9: score MMA issue (rank 0), TMEM allocation
constexpr int kMlaPvIssuer = 10;          // warp 10: value MMA issue (rank 0)
constexpr int kMlaThreads = 32 * (kMlaSoftmaxWarps + 3);
constexpr int kMlaTok = kMlaHalf / 2;     // tokens of a tile per softmax thread
constexpr int kMlaRescale = 8;            // raise the running max only past 2^8 growth
#ifndef PA_MLA_SEQ_UNITS
#define PA_MLA_SEQ_UNITS 2
#endif
constexpr int kMlaSeqUnits = PA_MLA_SEQ_UNITS;   // work units counted per sequence besides its tiles
#ifndef PA_MLA_PV_FIRST
#define PA_MLA_PV_FIRST 1
#endif
// Tensor-pipe order (1): the score MMA of tile m is issued only after both passes of
// the value MMA of tile m - 2, so that a tile's value MMA does not queue behind the
// score MMA of the tile after next (0: each stream issues as soon as it may)
constexpr bool kMlaPvFirst = PA_MLA_PV_FIRST != 0;

struct MlaParams {
  const uint16_t *q;            // [B][128][576]
  const uint16_t *lat;          // [nb * bs][576] latent rows (L2 prefetches)
  const int32_t *block_table;   // [B][mbs]
  const int32_t *context_lens;  // [B]
  void *out;                    // [B][128][512] bf16
  float *part_o;                // [slots][128][512]
  float *part_lse;              // [slots][128], log2 units
  int B, bs, mbs, nb;
  int parts;                    // pieces (CTA pairs)
  int min_tiles;                // > 0: at least this many tiles per piece (automatic launches)
  float scale_log2;
};

struct MlaLayout {
  static constexpr int kSlab = kMlaHalf * 128;            // 48 rows x 64 bf16 = 6 KB
  static constexpr int kSlabs = kMlaDk / 64;              // 9 slabs per staged half tile
  static constexpr int kStage = kSlabs * kSlab;           // 54 KB
  static constexpr int kHSlab = 64 * 128;                 // 64 head rows x 64 bf16 = 8 KB
  static constexpr int kQSlabs = 4;                       // query dims [320, 576)
  static constexpr int stage = 0;
  static constexpr int qs = stage + kMlaStages * kStage;
  // P pool (64 head rows each, K-major, 128-byte swizzle): slab 0 = P hi of tokens
  // [0, 64), slab 2 = P lo of tokens [0, 64), slab 1 = P hi of tokens [64, 96) in
  // its first 64 bytes of every row and P lo of the same tokens in the last 64
  static constexpr int ps = qs + kQSlabs * kHSlab;
  static constexpr int bars = ps + 3 * kHSlab;
  static constexpr int nbars = 23;
  static constexpr int xch = bars + nbars * 8;            // float xm[2][2][128], xl[2][128]
  static constexpr int misc = xch + 6 * 128 * 4;         // tmem base, abort, scan, start
  static constexpr int end = misc + 128;
  static constexpr size_t bytes() { return 1024 + end; }
  static_assert(kStage % 1024 == 0 && kSlab % 1024 == 0 && qs % 1024 == 0 && ps % 1024 == 0,
                "swizzled tiles need 1 KB alignment");
};
static_assert(MlaLayout::bytes() <= 232448, "shared memory per CTA");

// Tensor memory columns (exactly 512, allocated for the pair)
constexpr int kTmS = 0;        // score buffers at 0 and 48: 48 columns each
constexpr int kTmQ = 96;       // query dims [0, 320): 20 k-steps x 8 columns
constexpr int kQTmemDims = 320;
constexpr int kTmO = 256;      // value accumulator: dims block 0 at 256, block 1 at 384
static_assert(kTmQ + kQTmemDims / 2 <= kTmO && kTmS + 2 * kMlaHalf <= kTmQ, "tensor memory map");

// tiles of 96 tokens in a sequence of c tokens (c clamped to [0, cap])
__device__ __forceinline__ int mla_tiles(int c, int cap) {
  return (min(max(c, 0), cap) + kMlaTile - 1) / kMlaTile;
}

// Walks the tiles of a piece in order: sequence b, tile j within it, its tile
// count P, and whether the tile opens / closes that sequence's run in the piece.
// 32 bytes from global memory through the non-coherent path (address 32-byte aligned).
__device__ __forceinline__ void ldg_v8(const void *src, uint32_t *r) {
  asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(src));
}

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

// Cache row of the 16-token box k (0..5: boxes 0-2 are the rank-0 CTA's half, 3-5
// the other's) of tile j of sequence b: -1 for a block id out of range, -2 for a
// box that lies wholly past the context (not loaded).
__device__ __forceinline__ int mla_box_row(const MlaParams &p, int b, int j, int k, int ctx) {
  const int t = j * kMlaTile + k * kMlaBox;
  if (t >= ctx) return -2;
  const int blk = __ldg(&p.block_table[static_cast<long long>(b) * p.mbs + t / p.bs]);
  if (blk < 0 || blk >= p.nb) return -1;
  return blk * p.bs + t % p.bs;
}

// Tokens of the tile's half `half` (0: the rank-0 CTA's 48, 1: the other's) that
// lie inside a context of ctx tokens.
__device__ __forceinline__ int mla_half_tokens(int ctx, int j, int half) {
  return min(max(ctx - j * kMlaTile - half * kMlaHalf, 0), kMlaHalf);
}

// barrier slots.  Local: each CTA waits on its own.  Pair: live in the rank-0
// CTA only (arrivals from both CTAs); the same slots are unused in the other.
enum MlaBar {
  kLatEmpty = 0,    // [3] local: the value MMA of the stage's tile is done (commit to both)
  kSFull = 3,       // [2] local: scores of tile n in the score buffer, slot n % 2 (commit
                    //     to both; one slot per parity so that no waiter is two phases behind)
  kOReady = 5,      // [2] local: value MMA of tile n done (commit to both, slot n % 2)
  kPvFull = 7,      // [3] local: the other CTA's tokens landed in this CTA's value slabs
  kQEmpty = 10,     // local: last score MMA of a sequence done (commit to both)
  kFinal = 11,      // local: every MMA done (one commit to both from each issuer)
  kStall = 12,      // local, test hook only: nothing ever arrives here
  kPhiFree = 13,    // local: the P hi pass of the value MMA is done (commit to both)
  kLatFull = 14,    // [3] pair: both CTAs' own tokens landed (2 arrivals + bytes)
  kPhiFull = 17,    // pair: P hi of the tile written, its value rows in place (16 warps)
  kQFull = 18,      // pair: query of a sequence in place in both CTAs (16 warps + 2 copies)
  kOFree = 19,      // pair: both epilogues have read the accumulator (16 warps)
  kPloFull = 20,    // pair: P lo of the tile written in both CTAs (16 warps)
  kSFree = 21       // [2] pair: both CTAs' softmax warps have read score buffer n % 2 (16 warps)
};

__global__ void __launch_bounds__(kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a32,
                  const __grid_constant__ CUtensorMap tm_w9, const __grid_constant__ CUtensorMap tm_w2,
                  const __grid_constant__ CUtensorMap tm_q, const MlaParams p) {
  using L = MlaLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::bars);
  float *xm = reinterpret_cast<float *>(sm + L::xch);            // [2][2][128] row maxima
  float *xl = xm + 4 * 128;                                        // [2][128] row sums
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(sm + L::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::misc + 4);
  volatile int *pv_issued = reinterpret_cast<volatile int *>(sm + L::misc + 8);   // value MMAs issued
  int *scan_scratch = reinterpret_cast<int *>(sm + L::misc + 16);   // [kMlaThreads / 32]
  int *start = reinterpret_cast<int *>(sm + L::misc + 64);          // b, j of the first tile, tiles

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = pair::rank();        // 0: issues the MMAs; heads [64 rank, +64)
  const int pc = blockIdx.x >> 1;            // which piece of the tile stream
  const int cap = p.mbs * p.bs;

  // ---- prologue (all threads).  The flattened work stream has, for every
  // non-empty sequence, kMlaSeqUnits empty units (its fixed cost: the query load
  // and the epilogue, measured at about two tiles' time) and then its tiles.  A
  // block-wide scan gives the piece [ub, ue) of the stream, the (sequence, tile) of
  // its first tile and its tile count.
  {
    const int per = (p.B + kMlaThreads - 1) / kMlaThreads;
    const int b0 = min(p.B, tid * per), b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) {
      const int c = __ldg(&p.context_lens[b]);
      if (blockIdx.x == 0 && (c < 0 || c > cap)) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
      local += seq_units(c, cap, kMlaTile, kMlaSeqUnits);
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
      start[2] = 0;
    }
    __syncthreads();
    int run = v - local, total = 0;
    for (int i = 0; i < kMlaThreads / 32; ++i) {
      if (i < warp) run += scan_scratch[i];
      total += scan_scratch[i];
    }
    const long long TU = total;
    const int pieces = used_pieces(p.parts, TU, p.min_tiles, p.B);
    const long long ub = pc < pieces ? piece_begin(pc, TU, pieces) : 0;
    const long long ue = pc < pieces ? piece_begin(pc + 1, TU, pieces) : 0;
    int cnt = 0;
    for (int b = b0; b < b1; ++b) {
      const int P = mla_tiles(__ldg(&p.context_lens[b]), cap);
      if (P == 0) continue;
      const long long t0 = run + kMlaSeqUnits, t1 = t0 + P;     // b's tile units
      if (run <= ub && ub < t1) {               // the sequence holding unit ub
        start[0] = b;
        start[1] = static_cast<int>(ub > t0 ? ub - t0 : 0);
      }
      const long long lo = ub > t0 ? ub : t0, hi = ue < t1 ? ue : t1;
      if (lo < hi) cnt += static_cast<int>(hi - lo);
      run += kMlaSeqUnits + P;
    }
    if (cnt > 0) atomicAdd(&start[2], cnt);
  }
  if (tid == 0) {
    for (int i = 0; i < L::nbars; ++i) {
      uint32_t cnt = 1;
      if (i >= kLatFull && i < kLatFull + kMlaStages) cnt = 2;
      if (i == kFinal) cnt = 2;           // the score issuer and the value issuer
      if (i == kPhiFull || i == kPloFull || i == kOFree || i == kSFree || i == kSFree + 1)
        cnt = 2 * kMlaSoftmaxWarps;
      if (i == kQFull) cnt = 2 * kMlaSoftmaxWarps + 2;   // + each CTA's query copy (with its bytes)
      mbar_init(&bar[i], cnt);
    }
    *abort_flag = 0;
    *pv_issued = 0;
    fence_barrier_init();
  }
  if (warp == kMlaIssuer) {
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

  const int ntiles = start[2];
  const int b_first = start[0], j_first = start[1];
  // the pair barriers, addressed in the rank-0 CTA
  const uint32_t phifull_pair = pair::map_to(&bar[kPhiFull], 0);
  const uint32_t sfree_pair0 = pair::map_to(&bar[kSFree], 0);
  const uint32_t sfree_pair1 = pair::map_to(&bar[kSFree + 1], 0);
  const uint32_t plofull_pair = pair::map_to(&bar[kPloFull], 0);
  const uint32_t qfull_pair = pair::map_to(&bar[kQFull], 0);
  const uint32_t ofree_pair = pair::map_to(&bar[kOFree], 0);
  // this CTA's value dims: latent slabs {2r, 2r+1, 4+2r, 5+2r}; the other CTA's
  // tokens for them are staged in the slabs of the same index xor 2
  const int vs0 = 2 * static_cast<int>(rank);

  if (warp == kMlaProducer) {
    // ------------------------------------------------------------ copy issue
    // Lane i holds the cache rows of the six 16-token boxes of tile wb + i
    // (current window) and wb + 32 + i (next window); lane 0 issues, whichever of
    // "own tokens of tile n" (stage free) and "other tokens of tile n" (scores of
    // tile n done) is ready first.  A box is 16 rows x 64 dims (2 KB) of one slab.
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
      prefetch_tensormap(&tm_a32);
      prefetch_tensormap(&tm_w9);
      prefetch_tensormap(&tm_w2);
    }
    // Copies of a CTA half (48 rows, the three 16-row groups at cache rows r[0..2],
    // -2 for a group past the context): a run of 48 contiguous rows (the half lies
    // in one block) moves as one 3-D box that lands as whole slabs; otherwise each
    // run of 32 or 16 contiguous rows moves as one 2-D box per slab.  The copy
    // engine takes about 17 boxes per microsecond per SM whatever their size, so
    // the box count, not the bytes, bounds small copies.
    auto run_of = [&](const int (&r)[kMlaBoxes], int k) {   // rows of the run starting at group k
      if (k == 0 && r[1] == r[0] + kMlaBox && r[2] == r[0] + 2 * kMlaBox) return 3;
      if (k < kMlaBoxes - 1 && r[k + 1] == r[k] + kMlaBox) return 2;
      return 1;
    };
    MlaCursor cur;
    cur.init(p, b_first, j_first, ntiles);
    // Cache rows of the tile's boxes held by this lane: this CTA's three (own, c/n
    // o*) and the other CTA's three (t*), for the current window (c) and the next (n)
    const int own_box = kMlaBoxes * static_cast<int>(rank), oth_box = kMlaBoxes - own_box;
    int c_o[kMlaBoxes], c_t[kMlaBoxes], n_o[kMlaBoxes], n_t[kMlaBoxes];
#pragma unroll
    for (int k = 0; k < kMlaBoxes; ++k) c_o[k] = c_t[k] = n_o[k] = n_t[k] = -2;
    auto look_up = [&](int base, int (&o)[kMlaBoxes], int (&t)[kMlaBoxes]) {
      const int n = min(32, ntiles - base);
      int mb = 0, mj = 0, mctx = 0;
      for (int i = 0; i < n; ++i, cur.next())
        if (lane == i) {
          mb = cur.b;
          mj = cur.j;
          mctx = cur.ctx;
        }
      const bool ok = lane < n;
#pragma unroll
      for (int k = 0; k < kMlaBoxes; ++k) {
        o[k] = ok ? mla_box_row(p, mb, mj, own_box + k, mctx) : -2;
        t[k] = ok ? mla_box_row(p, mb, mj, oth_box + k, mctx) : -2;
      }
    };
    int wb = 0;                      // first tile of the current window
    if (ntiles > 0) look_up(0, c_o, c_t);
    if (ntiles > 32) look_up(32, n_o, n_t);
    // rows of tile n's boxes (all lanes call): own (oth = false) or the other CTA's
    auto rows_of = [&](int n, bool oth, int (&r)[kMlaBoxes]) {
      const bool w = n - wb >= 32;
#pragma unroll
      for (int k = 0; k < kMlaBoxes; ++k) {
        const int v = oth ? (w ? n_t[k] : c_t[k]) : (w ? n_o[k] : c_o[k]);
        r[k] = __shfl_sync(0xffffffffu, v, (n - wb) & 31);
      }
    };
    int n_own = 0, n_pv = 0;
    uint64_t t_idle = globaltimer();
    uint32_t spins = 0;
    while (n_pv < ntiles && !aborted) {
      // slide the windows once the other-token loads have left the current one
      if (n_pv >= wb + 32) {
#pragma unroll
        for (int k = 0; k < kMlaBoxes; ++k) {
          c_o[k] = n_o[k];
          c_t[k] = n_t[k];
        }
        wb += 32;
        if (ntiles > wb + 32) look_up(wb + 32, n_o, n_t);
      }
      int act = 0;
      if (lane == 0) {
        // own tokens run at most one tile ahead of the next other-token fetch: the
        // fetch (an L2 hit that the value MMA waits on) queues behind this SM's
        // copies in flight, so fewer of them ahead of it means a shorter wait
        if (n_own < ntiles && n_own < n_pv + kMlaLookahead &&
            (n_own < kMlaStages ||
             mbar_test(&bar[kLatEmpty + n_own % kMlaStages], ((n_own / kMlaStages) & 1) ^ 1)))
          act = 1;
        if (n_pv < n_own && mbar_test(&bar[kSFull + n_pv % 2], (n_pv / 2) & 1))
          act = 2;                       // the other CTA's tokens first: the value MMA waits on them
      }
      act = __shfl_sync(0xffffffffu, act, 0);
      if (act == 1) {
        const int n = n_own++;
        const int st = n % kMlaStages;
        int r[kMlaBoxes];
        rows_of(n, false, r);
        if (lane == 0) {
          int boxes = 0;
#pragma unroll
          for (int k = 0; k < kMlaBoxes; ++k) {
            if (r[k] == -1) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
            boxes += r[k] >= 0;
          }
          const uint32_t full = pair::map_to(&bar[kLatFull + st], 0);
          pair::arrive_expect_tx_remote(full, L::kSlabs * kMlaBox * 128 * boxes);
          uint8_t *dst = sm + L::stage + st * L::kStage;
          for (int k = 0; k < kMlaBoxes;) {
            const int len = r[k] >= 0 ? run_of(r, k) : 1;
            if (r[k] >= 0 && len == 3) {
              pair::tma_load_3d_to_pair_bar(dst, &tm_w9, full, 0, r[k], 0, pol_keep);
            } else if (r[k] >= 0) {
#pragma unroll 1
              for (int sl = 0; sl < L::kSlabs; ++sl)
                pair::tma_load_2d_to_pair_bar(dst + sl * L::kSlab + k * kMlaBox * 128,
                                              len == 2 ? &tm_a32 : &tm_a, full, 64 * sl, r[k],
                                              pol_keep);
            }
            k += len;
          }
        }
        // Pull the own rows of the tile kMlaPrefetch ahead into L2 (kept there): its
        // copy, issued once a stage frees, then reads L2 instead of waiting on HBM
        // behind this SM's other copies.  One bulk prefetch per contiguous run.
        if (kMlaPrefetch > 0 && n + kMlaPrefetch < ntiles) {
          int f[kMlaBoxes];
          rows_of(n + kMlaPrefetch, false, f);
          if (lane == 0)
            for (int k = 0; k < kMlaBoxes;) {
              const int len = f[k] >= 0 ? run_of(f, k) : 1;
              if (f[k] >= 0)
                prefetch_l2_bulk(p.lat + static_cast<long long>(f[k]) * kMlaDk,
                                 len * kMlaBox * kMlaDk * 2, pol_keep);
              k += len;
            }
        }
      } else if (act == 2) {
        const int n = n_pv++;
        const int st = n % kMlaStages;
        int r[kMlaBoxes];
        rows_of(n, true, r);
        if (lane == 0) {
          int boxes = 0;
#pragma unroll
          for (int k = 0; k < kMlaBoxes; ++k) boxes += r[k] >= 0;
          mbar_arrive_expect_tx(&bar[kPvFull + st], 4 * kMlaBox * 128 * boxes);
          // the value dims: latent slabs vs0, vs0 + 1, vs0 + 4, vs0 + 5, into the
          // stage's slabs of index xor 2
          uint8_t *dst = sm + L::stage + st * L::kStage;
          for (int k = 0; k < kMlaBoxes;) {
            const int len = r[k] >= 0 ? run_of(r, k) : 1;
            if (r[k] >= 0 && len == 3) {
              // two 64 dims x 48 rows x 2 slabs boxes (slab pairs vs0, vs0 + 1 and
              // vs0 + 4, vs0 + 5 into the pairs of index xor 2)
#pragma unroll
              for (int g = 0; g < 2; ++g)
                tma_load_3d_hint(dst + ((vs0 + 4 * g) ^ 2) * L::kSlab, &tm_w2, &bar[kPvFull + st],
                                 0, r[k], vs0 + 4 * g, pol_once);
            } else if (r[k] >= 0) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int sl = vs0 + (i & 1) + 4 * (i >> 1);
                tma_load_2d_hint(dst + (sl ^ 2) * L::kSlab + k * kMlaBox * 128,
                                 len == 2 ? &tm_a32 : &tm_a, &bar[kPvFull + st], 64 * sl, r[k],
                                 pol_once);
              }
            }
            k += len;
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
  } else if (warp == kMlaIssuer || warp == kMlaPvIssuer) {
    // ------------------------------------------------------------ MMA issuers (rank 0)
    // One thread issues the score MMAs and another the value MMAs, each with its own
    // commits, so that a tile's value MMA is not queued behind the issue of the next
    // tile's score MMAs.  The two streams share no tensor or shared memory they
    // write; every order between them runs through the barriers below.
    const bool s_role = warp == kMlaIssuer;
    if (rank == 0 && lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kMlaTile, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, 256, true);
      // descriptors are a base descriptor plus the byte offset / 16 (address field
      // in the low bits); every offset added below is a compile-time constant
      const uint64_t b_desc0 = umma_desc(smem_u32(sm + L::stage), 16, 1024);        // K-major
      const uint64_t v_desc0 = umma_desc(smem_u32(sm + L::stage), L::kSlab, 1024);  // MN-major
      const uint64_t q_desc0 = umma_desc(smem_u32(sm + L::qs), 16, 1024);
      const uint64_t p_desc0 = umma_desc(smem_u32(sm + L::ps), 16, 1024);
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
        const uint32_t d = tmem + kTmS + (n % 2) * kMlaHalf;
        // 16-dim step ks reads latent slab ks/4 at byte offset 32 (ks%4) of each row;
        // the query's first 320 dims come from tensor memory, the rest from its
        // shared-memory slabs
#pragma unroll
        for (int ks = 0; ks < kMlaDk / 16; ++ks) {
          const uint64_t b = bst + (((ks >> 2) * L::kSlab + (ks & 3) * 32) >> 4);
          if (ks < kQTmemDims / 16) {
            pair::mma_ts(d, tmem + kTmQ + ks * 8, b, idesc_s, ks > 0);
          } else {
            const int kq = ks - kQTmemDims / 16;
            pair::mma_ss(d, q_desc0 + (((kq >> 2) * L::kHSlab + (kq & 3) * 32) >> 4), b, idesc_s,
                         true);
          }
        }
        pair::commit_both(&bar[kSFull + n % 2]);
        if (last) pair::commit_both(&bar[kQEmpty]);
      };
      // The value MMA of tile n in two passes: P hi (written as soon as the softmax
      // is done), then P lo.  Dims block nb: the CTAs supply dims [256nb, 256nb+128)
      // and [256nb+128, 256nb+256); token half h of the tile sits in slabs
      // 4nb + 2h, 4nb + 2h + 1 of both CTAs (own tokens or the other CTA's, see
      // above); 16 tokens (2 KB of each slab) per step.  P's 16 tokens from t0 on
      // lie in pool slab 0 (hi) or 2 (lo) for t0 < 64, else in slab 1 (hi in the
      // first 64 bytes of a row, lo in the last 64).
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
            for (int kq = 0; kq < kMlaBoxes; ++kq) {
              const int t0 = kMlaHalf * h + 16 * kq;
              const int poff = t0 < 64 ? (lo_pass ? 2 : 0) * L::kHSlab + 2 * t0
                                       : L::kHSlab + (lo_pass ? 64 : 0) + 2 * (t0 - 64);
              const uint64_t a = p_desc0 + (poff >> 4);
              const uint64_t b = vb + ((kq * 2048) >> 4);
              pair::mma_ss(tmem + kTmO + nb * 128, a, b, idesc_o,
                           lo_pass || !(first && h == 0 && kq == 0));
            }
          }
        }
        if (lo_pass) {
          pair::commit_both(&bar[kLatEmpty + st]);
          pair::commit_both(&bar[kOReady + n % 2]);
        } else {
          pair::commit_both(&bar[kPhiFree]);
        }
      };
      // S(m) once both CTAs' softmax warps have read S(m-2) out of score buffer
      // m % 2, both CTAs' own tokens of tile m have landed, at a sequence start the
      // query is in place, and PVlo(m-2) has been issued.  PVhi(m) once P hi is
      // written and the value rows are in place in both CTAs and, at a sequence
      // start, the previous O has been read out; PVlo(m) once P lo is written.  Each
      // stream in tile order.
      int ns = 0, nh = 0, nl = 0;
      uint64_t t_idle = globaltimer();
      uint32_t spins = 0;
      while (s_role ? ns < ntiles : nl < ntiles) {
        bool did = false;
        if (s_role) {
          if ((ns < 2 || pair::test_cluster(&bar[kSFree + ns % 2], ((ns / 2) & 1) ^ 1)) &&
              pair::test_cluster(&bar[kLatFull + ns % kMlaStages], (ns / kMlaStages) & 1) &&
              (!cs.first() || pair::test_cluster(&bar[kQFull], (s_seg + 1) & 1)) &&
              (!kMlaPvFirst || ns < 2 || *pv_issued >= ns - 1)) {
            issue_s(ns++);
            did = true;
          }
        } else {
          if (nh < ntiles && pair::test_cluster(&bar[kPhiFull], nh & 1) &&
              (!cp.first() || o_seg < 0 || pair::test_cluster(&bar[kOFree], o_seg & 1))) {
            issue_pv(nh++, false);
            did = true;
          }
          if (nl < nh && pair::test_cluster(&bar[kPloFull], nl & 1)) {
            issue_pv(nl++, true);
            *pv_issued = nl;             // both passes of tile nl - 1 are in the pipe
            did = true;
          }
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
    // every MMA issued has completed before tensor memory is released (each issuer
    // commits once; one with nothing to do commits at once)
    if (rank == 0 && lane == 0) pair::commit_both(&bar[kFinal]);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue (warps 0-7)
    // Warp w reads TMEM lanes [32 (w % 4), +32) (the lanes a warp may access) and
    // column group cg = w / 4 of them.  A head's row of scores lies in lanes l and
    // 64 + l (token halves), and each lane's 48 columns are split between the two
    // column groups: cg 0 takes columns [0, 16) and [32, 40), cg 1 [16, 32) and
    // [40, 48) (loads of 16 and 8 columns at offsets aligned to their size).  So
    // four threads share a head: (hh, cg), in warps w, w + 2, w + 4, w + 6.
    const int t = tid;
    const int cg = warp >> 2;                          // column group
    const int tl = 32 * (warp & 3) + lane;             // TMEM lane
    const int lh = tl & 63;                            // head 64 rank + lh
    const int hh = tl >> 6;                            // token half of each tile
    const int head = 64 * static_cast<int>(rank) + lh;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    // the thread's tokens: 8-token chunks {2 cg, 2 cg + 1, 4 + cg} of its half
    auto chunk_of = [&](int i) { return i < 2 ? 2 * cg + i : 4 + cg; };
    bool aborted = false;

    // Query of sequence b.  Dims [320, 576) of the CTA's 64 heads land in shared
    // memory with one copy (a 64 dims x 64 rows x 4 slabs box: the 128-byte
    // swizzled K-major layout of the A operand), counted on the rank-0 CTA's
    // query barrier.  Dims [0, 320) go into TMEM lane t as bf16 pairs (both lanes
    // of the head: the layout of a 2-SM A operand), each column group taking half
    // of them in two batches.  Called after the previous sequence's last score MMA.
    auto load_query = [&](int b) {
      if (t == 0) {
        pair::arrive_expect_tx_remote(qfull_pair, L::kQSlabs * L::kHSlab);
        pair::tma_load_3d_to_pair_bar(sm + L::qs, &tm_q, qfull_pair, 0,
                                      b * kMlaHeads + 64 * static_cast<int>(rank),
                                      kQTmemDims / 64, l2_evict_first_policy());
      }
      const uint16_t *row = p.q + (static_cast<long long>(b) * kMlaHeads + head) * kMlaDk;
      // 32-byte loads where the query allows (rows are 1152 bytes apart), else 16
      const bool wide = (reinterpret_cast<uintptr_t>(p.q) & 31u) == 0;
      // column group cg writes TMEM columns [80 cg, 80 cg + 80) (dims [160 cg, +160))
      // in two batches, 32 + 48 columns (cg 0) or 48 + 32 (cg 1), every load of a
      // batch issued before its stores
      auto batch = [&](int col, auto ncols_c) {
        constexpr int NC = decltype(ncols_c)::value;   // 32 or 48
        uint32_t v[NC];
        if (wide) {
#pragma unroll
          for (int i = 0; i < NC / 8; ++i) ldg_v8(row + 2 * col + 16 * i, v + 8 * i);
        } else {
          const uint4 *src = reinterpret_cast<const uint4 *>(row + 2 * col);
#pragma unroll
          for (int i = 0; i < NC / 4; ++i) {
            const uint4 x = __ldg(src + i);
            v[4 * i] = x.x;
            v[4 * i + 1] = x.y;
            v[4 * i + 2] = x.z;
            v[4 * i + 3] = x.w;
          }
        }
        auto st32 = [&](int c, int o) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = v[o + i];
          tmem_st32u(tmem + kTmQ + c + lane_off, w);
        };
        auto st16 = [&](int c, int o) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = v[o + i];
          tmem_st16u(tmem + kTmQ + c + lane_off, w);
        };
        if constexpr (NC == 32) {
          st32(col, 0);
        } else if (col % 32 == 0) {
          st32(col, 0);
          st16(col + 32, 32);
        } else {
          st16(col, 0);
          st32(col + 16, 16);
        }
      };
      if (cg == 0) {
        batch(0, std::integral_constant<int, 32>());
        batch(32, std::integral_constant<int, 48>());
      } else {
        batch(80, std::integral_constant<int, 48>());
        batch(128, std::integral_constant<int, 32>());
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::arrive_remote(qfull_pair);
    };

    // Pull the query of sequence b into L2 a tile ahead of load_query, marked to
    // stay (the latent tiles streaming meanwhile are marked the same way): the
    // TMEM part (dims [0, 320): five 128-byte lines, shared by the head's two
    // threads)
    // and the shared-memory part's box.
    const uint64_t pol_q = l2_evict_last_policy();
    auto prefetch_query = [&](int b) {
      if (b < 0 || b >= p.B) return;
      const char *row = reinterpret_cast<const char *>(
          p.q + (static_cast<long long>(b) * kMlaHeads + head) * kMlaDk);
      for (int i = hh + 2 * cg; i < kQTmemDims * 2 / 128; i += 4)
        asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(row + i * 128));
      if (t == 0)
        tma_prefetch_3d(&tm_q, 0, b * kMlaHeads + 64 * static_cast<int>(rank), kQTmemDims / 64,
                        pol_q);
    };

    // Zero rows [from, 48) of the four slabs at slab indices first, first + 1,
    // first + 4, first + 5 of a stage (value rows of tokens past a ragged end, so
    // that 0 x stale data stays 0); the softmax threads share the work.
    auto zero_rows = [&](uint8_t *stage, int first, int from) {
      const int rows = kMlaHalf - from;
      for (int i = t; i < rows * 4 * 8; i += 32 * kMlaSoftmaxWarps) {
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
      float sc[kMlaTok];
      {
        const bool got = !aborted && mbar_wait(&bar[kSFull + n % 2], (n / 2) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        const uint32_t scol = tmem + kTmS + (n % 2) * kMlaHalf + lane_off;
        float (&s0)[16] = *reinterpret_cast<float (*)[16]>(&sc[0]);
        float (&s1)[8] = *reinterpret_cast<float (*)[8]>(&sc[16]);
        tmem_ld16(scol + 16 * cg, s0);
        tmem_ld8(scol + 32 + 8 * cg, s1);
        tmem_wait_ld();
        // the score buffer is free for the next tile's score MMA
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pair::arrive_remote(n % 2 ? sfree_pair1 : sfree_pair0);
      }
      // ---- online softmax (log2 units); the head's four threads agree on the max
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kMlaTok; ++i) {
        sc[i] = 8 * chunk_of(i / 8) + i % 8 < ntok ? sc[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, sc[i]);
      }
      {
        float *x = xm + (n & 1) * 256;
        x[cg * 128 + tl] = mt;
        named_bar_sync(1 + (warp & 1), 128);   // warps w, w + 2, w + 4, w + 6 hold the same heads
        mt = fmaxf(fmaxf(mt, x[cg * 128 + (tl ^ 64)]),
                   fmaxf(x[(1 - cg) * 128 + tl], x[(1 - cg) * 128 + (tl ^ 64)]));
      }
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
        for (int c = 128 * cg; c < 128 * cg + 128; c += 32) {
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
      // A operand of the value MMA: heads x 96 tokens, K-major, 128-byte swizzle;
      // 16-byte chunk c of a row holds tokens 48 hh + 8c .. + 7 (pool slabs: see
      // the layout), and this thread writes chunks chunk_of(0..2)
      uint32_t hi[kMlaTok / 2], lo[kMlaTok / 2];
#pragma unroll
      for (int e = 0; e < kMlaTok / 2; ++e) {
        const float p0 = ex2_approx(sc[2 * e] - m_run);
        const float p1 = ex2_approx(sc[2 * e + 1] - m_run);
        split2<true>(p0, p1, hi[e], lo[e]);
        l_run += p0 + p1;
      }
      // where chunk c of P goes: pool slab and 16-byte column of row lh
      auto p_chunk = [&](int c, bool lo_copy) {
        const int tk = kMlaHalf * hh + 8 * c;
        const int slab = tk < 64 ? (lo_copy ? 2 : 0) : 1;
        const int col = tk < 64 ? tk / 8 : (lo_copy ? 4 : 0) + (tk - 64) / 8;
        return sm + L::ps + slab * L::kHSlab + lh * 128 + ((col ^ (lh & 7)) << 4);
      };
      // P hi: its single buffer is released by the previous tile's hi pass
      if (n > 0) {
        const bool got = !aborted && mbar_wait(&bar[kPhiFree], (n - 1) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
      }
#pragma unroll
      for (int c = 0; c < kMlaTok / 8; ++c)
        *reinterpret_cast<uint4 *>(p_chunk(chunk_of(c), false)) =
            make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
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
#pragma unroll
      for (int c = 0; c < kMlaTok / 8; ++c)
        *reinterpret_cast<uint4 *>(p_chunk(chunk_of(c), true)) =
            make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
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
        xl[cg * 128 + tl] = l_run;
        named_bar_sync(1 + (warp & 1), 128);
        const float l_tot = (l_run + xl[cg * 128 + (tl ^ 64)]) +
                            (xl[(1 - cg) * 128 + tl] + xl[(1 - cg) * 128 + (tl ^ 64)]);
        // the sequence's tiles all lie in this piece iff it starts and ends inside
        const bool whole = n - j >= 0 && n - j + P <= ntiles;
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        const long long slot = pc + b;
        // The rows leave through shared memory: a thread's row would spread each
        // store instruction over 32 lines.  Warp w stages its 32 rows (TMEM lanes
        // 32 (w % 4) + r, heads 64 rank + (32 (w % 4) + r) % 64) 64 bytes at a time in
        // its 2 KB of the P pool, 16-byte chunk k of row r at chunk k ^ ((r >> 1) & 3),
        // and stores 8 rows x 64 contiguous bytes per instruction.  The pool is free:
        // the sequence's last value MMA is done, and the next tile's P is written
        // after the barrier that ends this epilogue.
        uint8_t *stg = sm + L::ps + warp * 2048;
        uint8_t *stg_w = stg + lane * 64;
        const int sw_w = (lane >> 1) & 3;
        const int rr = lane >> 2, kk = lane & 3;
        auto stage_row = [&](const uint4 (&w)[4]) {
          __syncwarp();                                  // the previous pass has been read
#pragma unroll
          for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4 *>(stg_w + 16 * (k ^ sw_w)) = w[k];
          __syncwarp();
        };
        auto staged = [&](int i) {                       // row 8 i + rr, chunk kk
          const int r = 8 * i + rr;
          return *reinterpret_cast<const uint4 *>(stg + r * 64 + 16 * (kk ^ ((r >> 1) & 3)));
        };
        auto head_of = [&](int i) {
          return 64 * static_cast<int>(rank) + ((32 * (warp & 3) + 8 * i + rr) & 63);
        };
#pragma unroll 1
        for (int c = 128 * cg; c < 128 * cg + 128; c += 32) {
          float v[32];
          tmem_ld32(tmem + kTmO + c + lane_off, v);
          tmem_wait_ld();
          // column c of dims block c / 128: dims 256 (c / 128) + 128 hh + c % 128
          const int d0 = 256 * (c >> 7) + 128 * hh + (c & 127);
          if (whole) {
            uint4 w[4];
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              w[q8].x = pack2<true>(v[8 * q8] * inv, v[8 * q8 + 1] * inv);
              w[q8].y = pack2<true>(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv);
              w[q8].z = pack2<true>(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv);
              w[q8].w = pack2<true>(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv);
            }
            stage_row(w);
            uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                          static_cast<long long>(b) * kMlaHeads * kMlaDv + d0 + 8 * kk;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4 *>(o + static_cast<long long>(head_of(i)) * kMlaDv) = staged(i);
          } else {
            float *o = p.part_o + slot * kMlaHeads * kMlaDv + d0 + 4 * kk;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint4 w[4];
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const float *x = v + 16 * half + 4 * q4;
                w[q4] = make_uint4(__float_as_uint(x[0] * inv), __float_as_uint(x[1] * inv),
                                   __float_as_uint(x[2] * inv), __float_as_uint(x[3] * inv));
              }
              stage_row(w);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4 *>(o + static_cast<long long>(head_of(i)) * kMlaDv + 16 * half) =
                    staged(i);
            }
          }
        }
        if (!whole && hh == 0 && cg == 0)
          p.part_lse[slot * kMlaHeads + head] = l_tot > 0.f ? m_run + log2f(l_tot) : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pair::arrive_remote(ofree_pair);
        // every softmax warp has read its staged rows before any writes the next P
        named_bar_sync(3, 32 * kMlaSoftmaxWarps);
      }
    }
  }

  // ---- teardown: every MMA of the pair has completed before either CTA frees
  // its tensor memory, and neither CTA leaves while the other may still signal it
  __syncthreads();
  if (warp == kMlaIssuer && lane == 0) {
    volatile int never = 0;
    mbar_wait(&bar[kFinal], 0, &never);
  }
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync();
  tc_fence_after();
  if (warp == kMlaIssuer)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace pa
