// pa_mla.cuh -- MLA (shared-latent) paged split-KV decode: the partition pass on
// the 5th-generation tensor cores (tcgen05, operands and accumulators in tensor
// memory).
//
// What it computes.  All H = 128 query heads of a sequence read one compressed
// latent vector per token (page "wenku.it search: Multi-head Latent Attention
// (MLA)", DeepSeek-V2 abstract on the latent KV): the key is the whole
// 576-wide latent row and the value its first 512 dims, so per sequence
//   out[h, :] = softmax_t(scale * q[h, :] . c_t) c_t[0:512].
// The KV stream is split and merged exactly as for GQA (page
// "cidian.kuaisou.com: flash decoding ++", three-step snippets): the flattened
// stream of 64-token tiles is cut into equal pieces, two CTAs per piece; a piece
// that covers a whole sequence writes the output, otherwise it leaves a
// normalised partial and the log-sum-exp of each head row for the merge kernel.
//
// Why two CTAs per piece.  The value accumulator O (128 heads x 512 fp32) alone
// fills the 512 columns of one SM's tensor memory, so a piece is run by two CTAs
// that each own half of the value dims:
//   CTA r accumulates O[:, 256r : 256r+256]                        (TMEM 256 columns)
// and both compute the whole score tile S = Q C^T (K = 576) themselves, so they
// never wait on each other: the same MMAs on the same operands give both CTAs
// bit-identical scores and hence identical P.  Recomputing S costs 36% more
// tensor work than splitting it, and buys the removal of every cross-SM
// exchange from the per-tile critical path.  The two CTAs read the same latent
// tiles at about the same time, so the second read is an L2 hit.
//
// Tile size.  One tcgen05.mma costs about 50 clocks to issue whatever its N, and
// an M=128 MMA reaches the tensor peak (~4K MAC/clock/SM) only from N = 128 up,
// so the score MMA (N = tokens per tile) wants big tiles; shared memory holds two
// 64-token latent stages (72 KB each) beside 80 KB of query.
//
// Operand placement.  As much of Q as fits sits in tensor memory (TS form, A
// from TMEM, so it costs no shared-memory bandwidth): dims [0, 256) in TMEM
// (128 columns), dims [256, 576) in shared memory (80 KB, the 128-byte swizzled
// K-major layout).
//
// Warp roles (192 threads).  Warps 0-3 own TMEM lanes 0-127 = head rows: they
// write the query into TMEM and shared memory per sequence, and per tile load
// the scores, run the online softmax in log2 units with a lazily raised running
// max, write P as a bf16 hi + lo pair over the tile's score columns, and at
// sequence ends normalise and store this CTA's half of O.  Warp 4 is the TMA
// producer (all 9 latent slabs of a tile as 32-row boxes, block table looked up
// 32 tiles ahead, 2-stage ring).  Warp 5 issues the MMAs from one thread, with
// every descriptor a base plus a compile-time offset:
//   S(n) = Q C^T   M=128 N=64  K=576  A in TMEM (256) + smem (320), B K-major
//   O   += P V_r   M=128 N=256 K=64 (x2: P hi, P lo)  A in TMEM, B MN-major
// S(m) and PV(m) are issued from one polling loop, whichever is ready first, so
// a value MMA never waits behind the load of a later tile.  Tiles are walked
// with cursors over context_lens (no per-sequence table in shared memory, so the
// batch size is not bounded by it).  All waits are bounded.
#pragma once

#include "pa_device.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

constexpr int kMlaTile = 64;              // tokens per tile
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
  int parts;                    // pieces (two CTAs each)
  int min_tiles;                // > 0: at least this many tiles per piece (automatic launches)
  float scale_log2;
};

struct MlaLayout {
  static constexpr int kLSlab = kMlaTile * 128;           // 64 rows x 64 bf16 = 8 KB
  static constexpr int kSlabs = kMlaDk / 64;              // 9 slabs per latent tile
  static constexpr int kStage = kSlabs * kLSlab;          // 72 KB
  static constexpr int kQSlab = kMlaHeads * 128;          // 128 rows x 64 bf16
  static constexpr int kQSmemDims = 320;                  // query dims [256, 576)
  static constexpr int stage = 0;
  static constexpr int qs = stage + kMlaStages * kStage;  // query dims [256, 576), 5 slabs
  static constexpr int bars = qs + (kQSmemDims / 64) * kQSlab;
  static constexpr int nbars = 16;
  static constexpr int misc = bars + nbars * 8;           // tmem base, abort, scan, start
  static constexpr int end = misc + 128;
  static constexpr size_t bytes() { return 1024 + end; }
  static_assert(kStage % 1024 == 0 && qs % 1024 == 0, "swizzled tiles need 1 KB alignment");
};
static_assert(MlaLayout::bytes() <= 232448, "shared memory per CTA");

// TMEM columns (exactly 512)
constexpr int kSBuf = 2;       // score / P buffers in flight
constexpr int kTmS = 0;        // buffers at 0, 64 (P hi in the first 32 columns, lo next 32)
constexpr int kTmQ = 128;      // query dims [0, 256): 128 columns (bf16 pairs)
constexpr int kQTmemDims = 256;
constexpr int kTmO = 256;      // value accumulator: 256 columns

// tiles of 64 tokens in a sequence of c tokens (c clamped to [0, cap])
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

// Cache row of the 32-token half h of tile j of sequence b: -1 for a block id
// out of range, -2 for a half that lies wholly past the context (not loaded).
__device__ __forceinline__ int mla_half_row(const MlaParams &p, int b, int j, int h, int ctx) {
  const int t = j * kMlaTile + h * kMlaBox;
  if (t >= ctx) return -2;
  const int blk = __ldg(&p.block_table[static_cast<long long>(b) * p.mbs + t / p.bs]);
  if (blk < 0 || blk >= p.nb) return -1;
  return blk * p.bs + t % p.bs;
}

// barrier slots
enum MlaBar {
  kLatFull = 0,     // [2] latent tile landed (TMA tx)
  kLatEmpty = 2,    // [2] both MMAs done with the stage (commit)
  kSFull = 4,       // [2] scores of tile n in buffer n%2 (commit)
  kPFull = 6,       // [2] P of tile n written into buffer n%2 (4 warps)
  kOReady = 8,      // [2] value MMA of tile n done (commit on slot n%2): with one slot
                    // per P buffer a waiter is never two phases behind, which a
                    // parity wait could not tell from being up to date
  kQFull = 10,      // query of sequence k in TMEM + shared memory (4 warps)
  kQEmpty = 11,     // last score MMA of sequence k done (commit)
  kOFree = 12,      // epilogue has read O (4 warps)
  kFinal = 13,      // all MMAs of this CTA done (commit)
  kStall = 14       // test hook only: nothing ever arrives here
};

__global__ void __launch_bounds__(kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_lat, const MlaParams p) {
  using L = MlaLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::bars);
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(sm + L::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::misc + 4);
  int *scan_scratch = reinterpret_cast<int *>(sm + L::misc + 16);   // [6]
  int *start = reinterpret_cast<int *>(sm + L::misc + 48);          // b, j of the first tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = blockIdx.x & 1;           // which half of the value dims
  const int pair = blockIdx.x >> 1;          // which piece of the tile stream
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
    tb = pair < pieces ? piece_begin(pair, TP, pieces) : 0;
    te = pair < pieces ? piece_begin(pair + 1, TP, pieces) : 0;
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
      if ((i >= kPFull && i < kPFull + kSBuf) || i == kQFull || i == kOFree) cnt = 4;
      mbar_init(&bar[i], cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_base_s))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = *tmem_base_s;
  // empty sequences: all-zero rows (the rank-0 CTA of each piece takes a share)
  if (rank == 0)
    for (int b = pair; b < p.B; b += p.parts)
      if (mla_tiles(__ldg(&p.context_lens[b]), cap) == 0)
        for (int i = tid; i < kMlaHeads * kMlaDv; i += kMlaThreads)
          reinterpret_cast<uint16_t *>(p.out)[static_cast<long long>(b) * kMlaHeads * kMlaDv + i] = 0;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int ntiles = static_cast<int>(te - tb);
  const int b_first = start[0], j_first = start[1];

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // Lane i looks up the two 32-row halves of tile base+i; lane 0 issues the
    // loads (18 boxes of 64 dims x 32 rows per tile) into the 2-stage ring.
    const uint64_t policy = l2_evict_first_policy();
    MlaCursor cur;
    cur.init(p, b_first, j_first, ntiles);
    int issued = 0;
    bool aborted = false;
    if (blockIdx.x == 0 && stall_test_enabled()) {
      // Test hook for the timeout path: wait, before anything is issued, on a
      // barrier that nothing completes.  The bounded wait gives up after about a
      // second, records PA_ERR_TIMEOUT and raises the CTA's abort flag, which
      // ends the issuer's and the softmax warps' waits too; no copy or MMA is in
      // flight, and tensor memory is released as usual.
      const bool got = lane != 0 || mbar_wait_idle(&bar[kStall], 0, abort_flag);
      aborted = !__all_sync(0xffffffffu, got);
    }
    if (lane == 0) prefetch_tensormap(&tm_lat);
    for (int base = 0; base < ntiles && !aborted; base += 32) {
      const int n = min(32, ntiles - base);
      // uniform walk (loads only at sequence changes), then the block-table
      // lookups of the whole batch in parallel, one tile per lane
      int mb = 0, mj = 0, mctx = 0;
      for (int i = 0; i < n; ++i, cur.next())
        if (lane == i) {
          mb = cur.b;
          mj = cur.j;
          mctx = cur.ctx;
        }
      int r0 = -2, r1 = -2;
      if (lane < n) {
        r0 = mla_half_row(p, mb, mj, 0, mctx);
        r1 = mla_half_row(p, mb, mj, 1, mctx);
      }
      for (int i = 0; i < n; ++i) {
        const int h0 = __shfl_sync(0xffffffffu, r0, i);
        const int h1 = __shfl_sync(0xffffffffu, r1, i);
        if (lane == 0 && !aborted) {
          const int nn = base + i;
          const int st = nn % kMlaStages;
          if (!mbar_wait_idle(&bar[kLatEmpty + st], ((nn / kMlaStages) & 1) ^ 1, abort_flag)) {
            aborted = true;
          } else if (h0 < 0 || h1 == -1) {
            record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
            mbar_arrive(&bar[kLatFull + st]);
            issued = nn + 1;
          } else {
            mbar_arrive_expect_tx(&bar[kLatFull + st],
                                  L::kSlabs * kMlaBox * 128 * (h1 >= 0 ? 2 : 1));
            uint8_t *dst = sm + L::stage + st * L::kStage;
            for (int s = 0; s < L::kSlabs; ++s) {
              tma_load_2d_hint(dst + s * L::kLSlab, &tm_lat, &bar[kLatFull + st], 64 * s, h0,
                               policy);
              if (h1 >= 0)
                tma_load_2d_hint(dst + s * L::kLSlab + kMlaBox * 128, &tm_lat,
                                 &bar[kLatFull + st], 64 * s, h1, policy);
            }
            issued = nn + 1;
          }
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && aborted) {
      volatile int never = 0;
      for (int nn = issued > kMlaStages ? issued - kMlaStages : 0; nn < issued; ++nn)
        mbar_wait(&bar[kLatFull + nn % kMlaStages], (nn / kMlaStages) & 1, &never);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kMlaTile, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, 256, true);
      // descriptors are a base descriptor plus the byte offset / 16 (address field
      // in the low bits); every offset added below is a compile-time constant
      const uint64_t b_desc0 = umma_desc(smem_u32(sm + L::stage), 16, 1024);       // K-major
      const uint64_t v_desc0 = umma_desc(smem_u32(sm + L::stage), L::kLSlab, 1024); // MN-major
      const uint64_t q_desc0 = umma_desc(smem_u32(sm + L::qs), 16, 1024);
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
        const uint32_t d = tmem + kTmS + (n % kSBuf) * kMlaTile;
        // 16-dim step ks reads latent slab ks/4 at byte offset 32 (ks%4) of each row
#pragma unroll
        for (int ks = 0; ks < kMlaDk / 16; ++ks) {
          const uint64_t b = bst + (((ks >> 2) * L::kLSlab + (ks & 3) * 32) >> 4);
          if (ks < kQTmemDims / 16) {
            umma_bf16_tmem_a(d, tmem + kTmQ + ks * 8, b, idesc_s, ks > 0);
          } else {
            const int kq = ks - kQTmemDims / 16;
            umma_bf16(d, q_desc0 + (((kq >> 2) * L::kQSlab + (kq & 3) * 32) >> 4), b, idesc_s, true);
          }
        }
        umma_commit(&bar[kSFull + n % kSBuf]);
        if (last) umma_commit(&bar[kQEmpty]);
      };
      auto issue_pv = [&](int n) {
        const int st = n % kMlaStages;
        const bool first = cp.first();
        cp.next();
        if (first) ++o_seg;
        tc_fence_after();
        const uint32_t pcol = tmem + kTmS + (n % kSBuf) * kMlaTile;
        // value dims [256r, 256r+256) of the stage, 16 tokens (2 KB) per step
        const uint64_t bv = v_desc0 + ((st * L::kStage + 4 * rank * L::kLSlab) >> 4);
#pragma unroll
        for (int kk = 0; kk < kMlaTile / 16; ++kk) {
          umma_bf16_tmem_a(tmem + kTmO, pcol + kk * 8, bv + kk * (2048 >> 4), idesc_o,
                           !(first && kk == 0));
          umma_bf16_tmem_a(tmem + kTmO, pcol + kMlaTile / 2 + kk * 8, bv + kk * (2048 >> 4),
                           idesc_o, true);
        }
        umma_commit(&bar[kLatEmpty + st]);
        umma_commit(&bar[kOReady + n % kSBuf]);
      };
      // S(m) and PV(m) are each issued in tile order, and whichever is ready goes
      // first: S(m) once PV(m-2) is issued (it reuses that P buffer; the tensor
      // pipe runs one thread's MMAs in order), its latent tile has landed and, at
      // a sequence start, the query is in place; PV(m) once P(m) is written and,
      // at a sequence start, the previous O has been read out.  A PV never waits
      // behind the load of a later tile.
      int ns = 0, npv = 0;
      uint64_t t_idle = globaltimer();
      uint32_t spins = 0;
      while (npv < ntiles) {
        bool did = false;
        if (ns < ntiles && ns < npv + kSBuf &&
            mbar_test(&bar[kLatFull + ns % kMlaStages], (ns / kMlaStages) & 1) &&
            (!cs.first() || mbar_test(&bar[kQFull], (s_seg + 1) & 1))) {
          issue_s(ns++);
          did = true;
        }
        if (npv < ns && mbar_test(&bar[kPFull + npv % kSBuf], (npv / kSBuf) & 1) &&
            (!cp.first() || o_seg < 0 || mbar_test(&bar[kOFree], o_seg & 1))) {
          issue_pv(npv++);
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
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(&bar[kFinal]);
      volatile int never = 0;
      mbar_wait(&bar[kFinal], 0, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue (warps 0-3)
    const int h = tid;                                   // head row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool aborted = false;

    // Query of sequence b: dims [0, 256) into TMEM row h as bf16 pairs (the layout
    // of a K-major A operand), dims [256, 576) into shared memory row h in the
    // 128-byte swizzled K-major layout (16-byte chunk c of a 128-byte row stored at
    // c ^ (h & 7)).  Called after the previous sequence's last score MMA is done.
    auto load_query = [&](int b) {
      const uint4 *src =
          reinterpret_cast<const uint4 *>(p.q + (static_cast<long long>(b) * kMlaHeads + h) * kMlaDk);
      // loads in batches of 16 x 16 bytes so that few round trips are serialised
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
      uint8_t *qrow = sm + L::qs + h * 128;
      constexpr int kQs = L::kQSmemDims / 64;          // 5 slabs: batches of 2, 2, 1
#pragma unroll 1
      for (int jq = 0; jq < kQs; jq += 2) {
        uint4 x[16];
        const int ns = min(2, kQs - jq);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < 8 * ns) x[i] = __ldg(src + kQTmemDims / 8 + jq * 8 + i);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < 8 * ns)
            *reinterpret_cast<uint4 *>(qrow + (jq + i / 8) * L::kQSlab + (((i & 7) ^ (h & 7)) << 4)) =
                x[i];
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kQFull]);
    };

    // Pull the query rows of sequence b into L2 ahead of load_query (fire and
    // forget: nine 128-byte lines per row).
    auto prefetch_query = [&](int b) {
      if (b < 0 || b >= p.B) return;
      const char *row =
          reinterpret_cast<const char *>(p.q + (static_cast<long long>(b) * kMlaHeads + h) * kMlaDk);
#pragma unroll
      for (int i = 0; i < kMlaDk * 2 / 128; ++i)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(row + i * 128));
    };

    // Before the query of the sequence starting at tile m may be written, the
    // score MMA of tile m-1 (the previous sequence's last) must have finished.
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
    // tile 0: its query is needed by the first score MMA
    if (ntiles > 0) {
      prefetch_query(b_first);
      prefetch_query(b_first + 1);
      query_for(0);
    }
    for (int n = 0; n < ntiles; ++n, cur.next()) {
      // S(n+1) can be issued once PV(n-1) is: give it its query now
      if (n + 1 < ntiles) query_for(n + 1);
      const int b = cur.b, j = cur.j, P = cur.P;
      const bool first = cur.first();
      const bool last = cur.last();
      if (first) {
        m_run = -INFINITY;
        l_run = 0.f;
        ctx = cur.ctx;
        if (n > 0) prefetch_query(b + 1);            // the sequence after this one
      }
      const int ntok = min(kMlaTile, ctx - j * kMlaTile);
      const int sb = n % kSBuf;
      const uint32_t scol = tmem + kTmS + sb * kMlaTile + lane_off;
      float sc[kMlaTile];
      {
        const bool got = !aborted && mbar_wait(&bar[kSFull + sb], (n / kSBuf) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        float (&s0)[32] = *reinterpret_cast<float (*)[32]>(&sc[0]);
        float (&s1)[32] = *reinterpret_cast<float (*)[32]>(&sc[32]);
        tmem_ld32(scol, s0);
        tmem_ld32(scol + 32, s1);
        tmem_wait_ld();
      }
      // ---- online softmax (log2 units), running max raised lazily
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kMlaTile; ++i) {
        sc[i] = i < ntok ? sc[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, sc[i]);
      }
      const bool raise = mt > m_run + kMlaRescale;
      if (__any_sync(0xffffffffu, raise && !first)) {
        // O must be scaled by 2^(m_old - m_new) for the rows whose max moved: wait
        // until the previous tile's value MMA has landed, then rescale in TMEM
        const bool got = !aborted && mbar_wait(&bar[kOReady + (n - 1) % kSBuf],
                                               ((n - 1) / kSBuf) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
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
      // ---- P = 2^(s - m) as a bf16 hi + lo pair (about 16 significant bits: a
      // single bf16 copy would bias the value mix by up to 2^-9 per weight),
      // written over this tile's score columns as the A operand of the value MMA:
      // hi pairs in the first 32 columns, lo pairs in the next 32
      {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < kMlaTile / 2; ++e) {
          const float p0 = ex2_approx(sc[2 * e] - m_run);
          const float p1 = ex2_approx(sc[2 * e + 1] - m_run);
          split2<true>(p0, p1, hi[e], lo[e]);
          l_run += p0 + p1;
        }
        tmem_st32u(scol, hi);
        tmem_st32u(scol + kMlaTile / 2, lo);
        tmem_wait_st();
      }
      // tokens past the end: zero their value rows so that 0 x stale data stays 0
      if (ntok < kMlaTile) {
        uint8_t *stg = sm + L::stage + (n % kMlaStages) * L::kStage;
        const int rows = kMlaTile - ntok;
        for (int i = h; i < rows * 4 * 8; i += kMlaHeads) {
          const int slab = i / (rows * 8), r = ntok + (i / 8) % rows, ch = i % 8;
          *reinterpret_cast<uint4 *>(stg + (4 * rank + slab) * L::kLSlab + r * 128 + ch * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kPFull + sb]);
      // ---- sequence end: normalise and write this CTA's half of the rows
      if (last) {
        const bool got = !aborted && mbar_wait(&bar[kOReady + sb], (n / kSBuf) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        // the sequence's tiles all lie in this piece iff it starts and ends inside
        const bool whole = n - j >= 0 && n - j + P <= ntiles;
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const long long slot = pair + b;
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld32(tmem + kTmO + c + lane_off, v);
          tmem_wait_ld();
          if (whole) {
            uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                          (static_cast<long long>(b) * kMlaHeads + h) * kMlaDv + rank * 256 + c;
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
            float *o = p.part_o + (slot * kMlaHeads + h) * kMlaDv + rank * 256 + c;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4 *>(o + 4 * q4) = make_float4(
                  v[4 * q4] * inv, v[4 * q4 + 1] * inv, v[4 * q4 + 2] * inv, v[4 * q4 + 3] * inv);
          }
        }
        if (!whole && rank == 0)
          p.part_lse[slot * kMlaHeads + h] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[kOFree]);
      }
    }
  }

  // ---- teardown: every MMA has completed (warp 5 waited for its final commit)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace pa
