// pa_gqa.cuh -- paged split-KV decode for grouped query heads (GQA / MHA / MQA):
// the partition pass.
//
// What it computes (page "cidian.kuaisou.com: flash decoding ++", snippets on the
// three Flash-Decoding steps): the KV stream of every (sequence, kv head) is cut
// into pieces along the sequence; for each piece and each of the G query heads
// that share the kv head, attention over the piece's tokens is computed with a
// running max and sum, and the piece's normalised output plus the log-sum-exp of
// its softmax row are recorded; the pieces are then rescaled by their
// log-sum-exps and reduced into the output.  A piece that covers a whole
// (sequence, kv head) writes the final output directly.
//
// How the pieces are chosen.  The KV stream is flattened into 16-token tiles in
// (sequence, kv head, tile) order, each non-empty (sequence, kv head) -- a
// "segment" -- preceded by seg_units empty units that stand for its fixed cost
// (query switch, output rows, the first tile's wait).  The stream is cut into P
// equal runs of units, one per warp of a persistent grid (P = CTAs x 8 warps;
// 12 in the float8 and index-list modes at up to 8 heads per group),
// so every warp carries the same work whatever the mix of context lengths.  A
// warp produces one result per segment whose tiles it touches.  The split
// points therefore fall where the work balances, not at a fixed length.
//
// Merge.  A warp that ends a segment it shares with other warps writes its
// normalised partial and log-sum-exp into slot (warp piece + segment); the merge
// kernel (pa_merge.cuh), launched right behind this one with programmatic
// dependent launch, combines them.  No barrier, fence or atomic is needed on
// the streaming path.  In the single-pass form (MODE 3) each piece counts itself
// in at its split segments once its last tile is done, and the last to arrive
// merges the segment.
//
// Data movement (the pages ask that K and V be loaded in parallel as fast as
// possible, then rescaled and combined).  Each warp is its own pipeline: lane 0
// issues TMA tensor copies (128-byte swizzle, L2 evict-first) of the next R
// tiles' K and V (16 x D each, physical block looked up through the block table
// by a 32-tile look-ahead held one tile per lane) into the warp's R-stage ring,
// each stage guarded by an mbarrier (at D 128 one 3-D box lands both 64-wide
// slabs of a tile).  Per tile the warp computes S^T = K Q^T with mma.sync
// m16n8k16 (tokens on M, the group's heads on N; two accumulators over the
// k-steps), the online softmax in registers (max over tokens with three xor
// shuffles, sums kept per lane) and O^T += V^T P with V^T fragments from
// ldmatrix.trans and P moved to the B operand layout with movmatrix (as a 16-bit
// hi + lo pair, two MMAs).  On the 16-bit TMA path the scores of tile t + 1 are
// taken before tile t's softmax, so each iteration holds two independent MMA
// chains.  The query fragments of the next segment are prefetched into registers.
//
// Float8 KV cache (KV8).  With E4M3 codes in the cache (one key scale and one
// value scale per tensor; page "bjpcjp.github.io: llms-attention",
// FlashAttention-3 teaser on FP8 low precision) the ring holds 1-byte tiles
// (one 16 x 128-byte TMA box for K and one for V, R = 6 stages).  The fragments
// are built straight from them: ldmatrix of the codes read as 16-bit pairs hands
// each lane four consecutive codes of one row (K) or, transposed, two dims x two
// tokens (V, paired per dim by one byte permute), and cvt.rn.f16x2.e4m3x2 widens
// them exactly (every E4M3 value is an fp16 value).  This fixes which head dims
// meet in a fragment: the query fragment takes the same dims, and the output
// rows are written back in dim order.  The MMAs then run in fp16 (a bf16 query
// is converted to fp16 once per segment; it must lie in the fp16 range).  The
// key scale is folded into the softmax scale and the value scale into the final
// 1 / l, so neither costs anything per token.
#pragma once

#include <type_traits>

#include "pa_device.cuh"
#include "pa_merge.cuh"

namespace pa {

constexpr int kTile = 16;               // tokens per pipeline tile
constexpr int kWarps = 8;               // independent streaming warps per CTA (default)
constexpr int kGqaThreads = 32 * kWarps;

// Warps per CTA of a kernel variant.  The float8 (1) and index-list (2) modes at
// up to 8 heads per group run 12: each of their warps is latency-bound (widening
// the codes; the lookup chain and row gathers), and 12 x 4 stages of 4 KB, or
// 12 x 2 stages of 8 KB, fill the same shared memory as 8 warps do.  Every other
// variant runs 8.
__host__ __device__ constexpr int gqa_warps(int mode, int nt) {
  return (mode == 1 || mode == 2) && nt == 1 ? 12 : kWarps;
}

struct GqaParams {
  const uint16_t *q;            // [B][Hq][D]
  const int32_t *block_table;   // [B][mbs]
  const int32_t *context_lens;  // [B]
  void *out;                    // [B][Hq][D] 16-bit
  float *part_o;                // [slots][G][D]
  float *part_lse;              // [slots][G], log2 units
  int B, Hq, Hkv, G, bs, mbs, nb;
  int tiles_per_block;          // bs / 16
  int parts;                    // gridDim.x
  float scale_log2;             // scale * log2(e)
  int min_tiles;               // > 0: at least this many tiles per piece (automatic launches)
  float v_scale;                // value scale of a float8 KV cache (1 otherwise)
  // index-list decode (MODE 2): context_lens holds the selected counts n_sel
  const int32_t *token_index;   // [B][max_sel] token positions
  int max_sel;
  const void *k_cache, *v_cache;  // the gathers read the caches directly
  // single-pass merge: nonzero epoch = the last piece of a split segment merges it
  unsigned long long *seg_ctr;  // [B * Hkv] arrival counters (epoch << 32 | count)
  uint32_t epoch;
  // Each non-empty segment's run of the flattened stream starts with seg_units
  // empty units, so that pieces are cut by tiles plus a fixed cost per segment
  int seg_units;
};

// MODE 0, 2 and 3: 16-bit rows in 128-byte swizzled slabs (2: gathered row by
// row into the same layout).  MODE 1: float8 rows.
template <int D, int NT, int R, int MODE = 0, int W = kWarps>
struct GqaLayout {
  static constexpr int kHeads = 8 * NT;            // group width padded to the MMA N
  static constexpr int kKTile = kTile * D * (MODE == 1 ? 1 : 2);  // bytes of one K (or V) tile
  static constexpr int kStage = 2 * kKTile;
  static constexpr int ring = 0;                   // warp w: stages [w*R, (w+1)*R)
  static constexpr int bars = ring + W * R * kStage;
  static constexpr int nbars = W * R;
  static constexpr int info = bars + nbars * 8;     // int stage_valid[W * R]
  static constexpr int flags = info + nbars * 4;    // abort flag + scan scratch
  static constexpr int prefix = flags + 64;         // int prefix[B + 1]
  static size_t bytes(int B) { return 1024 + prefix + static_cast<size_t>(B + 1) * 4; }
  static_assert(kStage % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(bars % 8 == 0, "mbarriers need 8-byte alignment");
};


// Segment (b, kvh) and tile j within it of flattened tile t (0 <= t < Hkv * prefix[B]).
__device__ __forceinline__ void locate_tile(const int *prefix, int B, int Hkv, long long t,
                                            int &b, int &kvh, int &j) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<long long>(Hkv) * prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  b = lo;
  const int P = prefix[b + 1] - prefix[b];
  const long long r = t - static_cast<long long>(Hkv) * prefix[b];
  kvh = static_cast<int>(r / P);
  j = static_cast<int>(r - static_cast<long long>(kvh) * P);
}

// Cache row of the first token of the tile at flattened unit t, -2 for one of a
// segment's leading empty units, or -1 if its block id is outside [0, nb)
// (recorded, never dereferenced).
__device__ __forceinline__ int tile_row(const GqaParams &p, const int *prefix, long long t) {
  int b, kvh, j;
  locate_tile(prefix, p.B, p.Hkv, t, b, kvh, j);
  j -= p.seg_units;
  if (j < 0) return -2;
  const int jb = j / p.tiles_per_block;
  const int blk = __ldg(&p.block_table[static_cast<long long>(b) * p.mbs + jb]);
  if (blk < 0 || blk >= p.nb) return -1;
  return (blk * p.Hkv + kvh) * p.bs + (j - jb * p.tiles_per_block) * kTile;
}

// Index-list decode: the lookups behind selected entry r (= lane % 16) of a
// tile form a three-step chain of dependent loads (count -> position -> block
// id).  Each step runs one tile apart, at successive issues, so every load has a
// tile's worth of time to land and no lane waits on one.
struct IdxLookup {
  int b3 = 0, kvh3 = 0, j3 = 0, n3 = 0, live3 = 0;   // located; count loading
  int b2 = 0, kvh2 = 0, pos2 = -2;                  // position loading (-2: none)
  int kvh1 = 0, pos1 = -2, blk1 = -1;               // block id loading (-1: bad)
};

// Advance the chain by one tile: the located tile moves on to its position load,
// the position to its block-id load, and tile t enters (live if t < end).
__device__ __forceinline__ void idx_advance(const GqaParams &p, const int *prefix, IdxLookup &k,
                                            long long t, long long end, int r) {
  k.kvh1 = k.kvh2;
  k.pos1 = k.pos2;
  if (k.pos2 >= 0 && k.pos2 < p.mbs * p.bs) {
    k.blk1 = __ldg(&p.block_table[static_cast<long long>(k.b2) * p.mbs + k.pos2 / p.bs]);
  } else {
    k.blk1 = -1;
    if (k.pos2 != -2) k.pos1 = -1;                  // a position outside the table
  }
  k.b2 = k.b3;
  k.kvh2 = k.kvh3;
  const int i = k.j3 * kTile + r;
  k.pos2 = (k.live3 && i < k.n3)
               ? __ldg(&p.token_index[static_cast<long long>(k.b3) * p.max_sel + i]) : -2;
  if (k.pos2 < 0 && k.pos2 != -2) k.pos2 = -1;
  k.live3 = t < end;
  if (k.live3) {
    locate_tile(prefix, p.B, p.Hkv, t, k.b3, k.kvh3, k.j3);
    k.n3 = __ldg(&p.context_lens[k.b3]);            // the selected count
    k.n3 = k.n3 < 0 ? 0 : (k.n3 > p.max_sel ? p.max_sel : k.n3);
  }
}

// Cache row of the tile at the end of the chain: -2 no entry, -1 bad (recorded
// by the caller, never dereferenced).
__device__ __forceinline__ int idx_row_of(const GqaParams &p, const IdxLookup &k) {
  if (k.pos1 == -2) return -2;
  if (k.pos1 < 0 || k.blk1 < 0 || k.blk1 >= p.nb) return -1;
  return (k.blk1 * p.Hkv + k.kvh1) * p.bs + k.pos1 % p.bs;
}

// Query B-operand fragments (Q^T: d x heads) of group (b, kvh): for n-tile nt and
// k-step ks, lane holds Q[head 8nt+g][16ks+2tq .. +1] and Q[..][16ks+8+2tq .. +1];
// heads past the group are zero.
// Two E4M3 code pairs (bytes 0,1 and bytes 2,3 of x) -> two fp16 pairs, exactly
// (every E4M3 value is an fp16 value).
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t x, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(x));
}

// bf16 pair -> fp16 pair (exact inside the fp16 range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xffff0000u);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// TO_F16: the query is bf16 and the MMAs run in fp16 (float8 KV cache).
// KV8: the float8 path feeds the score MMA's k-step ks with head dims
// 16 ks + 4 tq + {0, 1} as fragment columns 2 tq, 2 tq + 1 and 16 ks + 4 tq + {2, 3}
// as columns 2 tq + 8, 2 tq + 9 (the order an 8-bit row arrives in, see the
// kernel); the query fragment takes the same dims.
template <int D, int NT, bool TO_F16 = false, bool KV8 = false>
__device__ __forceinline__ void load_q(const GqaParams &p, int b, int kvh, int lane,
                                       uint32_t (&qf)[NT][D / 16][2]) {
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = nt * 8 + g;
    const bool ok = h < p.G;
    const uint32_t *row = reinterpret_cast<const uint32_t *>(
        p.q + (static_cast<long long>(b) * p.Hq + kvh * p.G + (ok ? h : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qf[nt][ks][0] = ok ? __ldg(row + ks * 8 + (KV8 ? 2 * tq : tq)) : 0u;
      qf[nt][ks][1] = ok ? __ldg(row + ks * 8 + (KV8 ? 2 * tq + 1 : 4 + tq)) : 0u;
      if (TO_F16) {
        qf[nt][ks][0] = bf16x2_to_f16x2(qf[nt][ks][0]);
        qf[nt][ks][1] = bf16x2_to_f16x2(qf[nt][ks][1]);
      }
    }
  }
}

// MODE 0: 16-bit cache, TMA tiles.  1: float8 cache (KV8).  2: index-list
// decode (IDX): each warp gathers its tiles' selected rows with cp.async.
// 3: as 0, and the last piece of each split segment merges it (FUSED).
template <int D, int NT, bool BF16, int R, int MODE = 0, int W = kWarps>
__global__ void __launch_bounds__(32 * W, 1)
gqa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const GqaParams p) {
  constexpr bool KV8 = MODE == 1, IDX = MODE == 2, FUSED = MODE == 3;
  // 16-bit TMA modes: the next tile's scores are taken ahead of this tile's
  // softmax (measured slower for the float8 and index-list modes)
  constexpr bool PIPE = !KV8 && !IDX;
  using L = GqaLayout<D, NT, R, MODE, W>;
  constexpr int kThreadsW = 32 * W;
  static_assert(W <= 12, "the scan scratch in the flags area holds 12 warps");
  static_assert(!KV8 || D == 128, "the float8 KV path reads 128-byte rows");
  static_assert(!IDX || D == 128, "index-list gathers read 256-byte rows");
  constexpr bool CT = BF16 && !KV8;          // MMA operand type: bf16, else fp16
  constexpr int KS = D / 16;                 // k-steps of the score MMA / m-tiles of the PV MMA

  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::flags);
  int *scan_scratch = reinterpret_cast<int *>(sm + L::flags) + 4;
  int *prefix = reinterpret_cast<int *>(sm + L::prefix);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int cap = IDX ? p.max_sel : p.mbs * p.bs;

  // Warm L2 with this CTA's share of the block table while the lengths load.
  {
    const char *tb = reinterpret_cast<const char *>(p.block_table);
    const long long bytes = static_cast<long long>(p.B) * p.mbs * 4;
    const long long lo = bytes * c / p.parts, hi = bytes * (c + 1) / p.parts;
    for (long long off = (lo & ~127ll) + tid * 128ll; off < hi; off += kThreadsW * 128ll)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(tb + off));
  }
  tiles_prefix<kThreadsW>(p.context_lens, p.B, cap, kTile, prefix, scan_scratch, c == 0,
                            p.seg_units);
  // let the merge grid be scheduled as SMs free up (it waits for this grid to finish)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // sequences with no tokens get an all-zero output row (spread over the grid)
  for (int b = c; b < p.B; b += p.parts)
    if (prefix[b + 1] == prefix[b])
      for (int i = tid; i < p.Hq * D; i += kThreadsW)
        reinterpret_cast<uint16_t *>(p.out)[static_cast<long long>(b) * p.Hq * D + i] = 0;

  const long long TP = static_cast<long long>(p.Hkv) * prefix[p.B];
  const int pieces = used_pieces(p.parts * W, TP, p.min_tiles,
                                 static_cast<long long>(W) * p.B * p.Hkv);
  const int gw = c * W + warp;                     // this warp's piece
  const long long wb = gw < pieces ? piece_begin(gw, TP, pieces) : 0;
  const long long we = gw < pieces ? piece_begin(gw + 1, TP, pieces) : 0;

  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::bars) + warp * R;
  int *stage_valid = reinterpret_cast<int *>(sm + L::info) + warp * R;
  uint8_t *ring = sm + L::ring + warp * R * L::kStage;
  if (lane == 0) {
    // IDX: 32 lanes' cp.async arrivals + lane 0's arrive after writing stage_valid
    for (int s = 0; s < R; ++s) mbar_init(&full[s], IDX ? 33 : 1);
    if (warp == 0) *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (wb >= we) return;

  bool aborted = false;
  if (c == 0 && warp == 0 && stall_test_enabled()) {
    // Test hook for the timeout path: wait on this warp's first stage barrier
    // before anything is issued into it, so that nothing can complete the wait.
    // The bounded wait gives up, records PA_ERR_TIMEOUT and raises the CTA's
    // abort flag.  The warp then runs its piece as aborted: it issues and waits
    // for nothing, and in the single-pass form it still counts itself in at its
    // split segments so that their counters return to zero.
    aborted = !__all_sync(0xffffffffu, mbar_wait(&full[0], 0, abort_flag));
  }

  const uint64_t policy = l2_evict_first_policy();
  if (lane == 0 && !IDX) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }

  // ---- look-ahead: lane i holds the cache row of tile la_base + i
  // (IDX: lane l holds the row of selected entry l % 16 of the next tile to issue)
  long long la_base = wb;
  int la_row = (!IDX && wb + lane < we) ? tile_row(p, prefix, wb + lane) : 0;
  long long nx_base = wb + 32;
  int nx_row = (!IDX && nx_base + lane < we) ? tile_row(p, prefix, nx_base + lane) : 0;
  IdxLookup idx;
  if (IDX)                               // fill the chain: tile wb at its end
    for (int x = 0; x < 3; ++x) idx_advance(p, prefix, idx, wb + x, we, lane & 15);
  long long issued = wb;                              // next tile to issue

  // Issue tile `issued` into its stage (lane 0 does the copy; all lanes call).
  auto issue_next = [&]() {
    if (issued >= we) return;
    if (IDX) {
      // gather: instruction x copies selected rows 2x and 2x + 1 whole, one per
      // half-warp, lane l taking 16-byte chunk l % 16 of its row (a row of K or V is
      // 256 contiguous bytes, so each copy instruction reads 4 full 128-byte
      // lines) into the swizzled layout the TMA path produces; lane r % 16 holds
      // the row index of entry r and shares it
      const long long n = issued - wb;
      const int st = static_cast<int>(n % R);
      const int idx_row = idx_row_of(p, idx);
      const bool bad = __any_sync(0xffffffffu, idx_row == -1);
      if (!bad) {
        const int ch = lane & 15, hw = lane >> 4;
        const uint32_t dk = smem_u32(ring + st * L::kStage), dv = dk + L::kKTile;
#pragma unroll
        for (int x = 0; x < kTile / 2; ++x) {
          const int r = 2 * x + hw;
          const int row = __shfl_sync(0xffffffffu, idx_row, r);
          if (row >= 0) {
            const long long off = static_cast<long long>(row) * D * 2 + ch * 16;
            const uint32_t so = sw128_offset(r, ch * 8, kTile);
            cp_async16(dk + so, static_cast<const char *>(p.k_cache) + off);
            cp_async16(dv + so, static_cast<const char *>(p.v_cache) + off);
          }
        }
      }
      cp_async_mbar_arrive_noinc(&full[st]);
      if (lane == 0) {
        if (bad) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
        stage_valid[st] = bad ? 0 : 1;
        mbar_arrive(&full[st]);
      }
      ++issued;
      idx_advance(p, prefix, idx, issued + 2, we, lane & 15);   // tile issued+2 enters
      return;
    }
    if (issued >= la_base + 32) {                     // slide the look-ahead window
      la_base = nx_base;
      la_row = nx_row;
      nx_base += 32;
      nx_row = (nx_base + lane < we) ? tile_row(p, prefix, nx_base + lane) : 0;
    }
    const int row = __shfl_sync(0xffffffffu, la_row, static_cast<int>(issued - la_base));
    const long long n = issued - wb;
    const int st = static_cast<int>(n % R);
    if (lane == 0) {
      if (row < 0) {                                  // bad block id, or an empty unit
        if (row == -1) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
        stage_valid[st] = 0;
        mbar_arrive(&full[st]);
      } else {
        stage_valid[st] = 1;
        mbar_arrive_expect_tx(&full[st], L::kStage);
        uint8_t *dst = ring + st * L::kStage;
        if (KV8) {                                    // one 16 x 128-byte box each
          tma_load_2d_hint(dst, &tm_k, &full[st], 0, row, policy);
          tma_load_2d_hint(dst + L::kKTile, &tm_v, &full[st], 0, row, policy);
        } else if (D == 128) {
          // one box per tile: the row's two 128-byte halves are the map's third
          // dimension, so the box lands as the two 64-wide swizzled slabs
          tma_load_3d_hint(dst, &tm_k, &full[st], 0, row, 0, policy);
          tma_load_3d_hint(dst + L::kKTile, &tm_v, &full[st], 0, row, 0, policy);
        } else {
#pragma unroll
          for (int x = 0; x < D; x += 64) {
            tma_load_2d_hint(dst + (x / 64) * kTile * 128, &tm_k, &full[st], x, row, policy);
            tma_load_2d_hint(dst + L::kKTile + (x / 64) * kTile * 128, &tm_v, &full[st], x, row,
                             policy);
          }
        }
      }
    }
    ++issued;
  };
  if (!aborted)
    for (int s = 0; s < R; ++s) issue_next();

  const int g = lane >> 2;          // fragment row group
  const int tq = lane & 3;          // thread in quad
  const uint32_t ring_base = smem_u32(ring);
  // per-lane ldmatrix row/column offsets (see the fragment layouts above)
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8, k_col = (lane >> 4) * 8;
  const int v_row = (lane & 7) + (lane >> 4) * 8, v_col = ((lane >> 3) & 1) * 8;

  // current and next segment
  int b, kvh, j0;
  locate_tile(prefix, p.B, p.Hkv, wb, b, kvh, j0);
  uint32_t qf[NT][KS][2], nq[NT][KS][2];
  load_q<D, NT, BF16 && KV8, KV8>(p, b, kvh, lane, qf);
  (void)tm_k;
  (void)tm_v;
  int ctx = clamp_ctx(__ldg(&p.context_lens[b]), cap);

  long long split_seg[2] = {0, 0}, split_first[2] = {0, 0};
  int split_tiles[2] = {0, 0}, n_split = 0;

  // float8: per-lane row address of the ldmatrix blocks of a 16 x 128-byte
  // tile (block j = lane / 8: tokens 8 (j & 1) .. +7, 16-byte chunk 2 x + j / 2)
  const int x8_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  auto x8_addr = [&](uint32_t tile, int x) {
    const int c = 2 * x + (lane >> 4);
    return tile + x8_row * 128 + ((c ^ (x8_row & 7)) << 4);
  };
  // scores S^T of the landed tile whose K starts at shared address kt
  auto scores = [&](uint32_t kt, float (&sc)[NT][4]) {
    // S^T (16 tokens x 8NT heads) = K Q^T, the k-steps alternating between two
    // accumulators (halves the chain of dependent MMAs), summed at the end
    float s2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = s2[nt][e] = 0.f;
    if (KV8) {
      // an ldmatrix block of 8 tokens x 16 codes gives lane (g, tq) the codes of
      // dims 4 tq .. 4 tq + 3 of token g: fragment columns (2tq, 2tq+1) and
      // (2tq+8, 2tq+9) after widening (the query matches, see load_q)
#pragma unroll
      for (int x = 0; x < KS / 2; ++x) {
        uint32_t r[4];
        ldsm_x4(x8_addr(kt, x), r);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t a[4];
          e4m3x4_to_f16x2(r[2 * h], a[0], a[2]);      // token g
          e4m3x4_to_f16x2(r[2 * h + 1], a[1], a[3]);  // token g + 8
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816<CT>(h ? s2[nt] : sc[nt], a, qf[nt][2 * x + h][0], qf[nt][2 * x + h][1]);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4];
        ldsm_x4(kt + sw128_offset(k_row, ks * 16 + k_col, kTile), a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816<CT>((ks & 1) ? s2[nt] : sc[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] += s2[nt][e];
  };
  // wait for the tile at position nn of the warp's run and take its scores
  // (zeros for a tile that did not land or was not loaded)
  auto land = [&](long long nn, float (&sc)[NT][4]) {
    const int sst = static_cast<int>(nn % R);
    const bool ok = !aborted && __all_sync(0xffffffffu, mbar_wait(&full[sst],
                                                                  static_cast<uint32_t>((nn / R) & 1),
                                                                  abort_flag));
    if (!ok) aborted = true;
    if (ok && stage_valid[sst]) {
      scores(ring_base + sst * L::kStage, sc);
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
    }
    return ok;
  };

  long long t = wb;
  while (t < we) {
    const int U = prefix[b + 1] - prefix[b];       // units of the segment
    const int P = U - p.seg_units;                 // its tiles
    const long long seg_first = static_cast<long long>(p.Hkv) * prefix[b] +
                                static_cast<long long>(kvh) * U;
    const long long tile_first = seg_first + p.seg_units;
    const long long seg_end = min(we, seg_first + U);
    // whole: every tile of the segment is in this piece (its output is written
    // here); has_tiles: this piece holds at least one of them
    const bool whole = tile_first >= wb && seg_first + U <= we;
    const bool has_tiles = seg_end > max(t, tile_first);
    // prefetch the next segment's query fragments and length
    int nb_ = b, nkvh = kvh, nj, nctx = ctx;
    if (seg_end < we) {
      locate_tile(prefix, p.B, p.Hkv, seg_end, nb_, nkvh, nj);
      load_q<D, NT, BF16 && KV8, KV8>(p, nb_, nkvh, lane, nq);
      nctx = clamp_ctx(__ldg(&p.context_lens[nb_]), cap);
    }

    float m[NT][2], l[NT][2], o[KS][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }

    // PIPE: tile t + 1's scores are taken before tile t's softmax and value MMA,
    // so each iteration holds two independent chains of MMAs.  Otherwise a tile
    // is waited for and scored in its own iteration.
    float s_cur[NT][4];
    bool ok_cur = PIPE ? land(t - wb, s_cur) : false;
    for (; t < seg_end; ++t) {
      const long long n = t - wb;
      const int st = static_cast<int>(n % R);
      float s_nxt[NT][4];
      bool ok_nxt = false;
      if (PIPE) {
        if (t + 1 < seg_end) ok_nxt = land(n + 1, s_nxt);
      } else {
        ok_cur = !aborted && __all_sync(0xffffffffu, mbar_wait(&full[st],
                                                               static_cast<uint32_t>((n / R) & 1),
                                                               abort_flag));
        if (!ok_cur) aborted = true;
      }
      const int jt = static_cast<int>(t - tile_first);
      const int ntok = (ok_cur && stage_valid[st]) ? min(kTile, ctx - jt * kTile) : 0;
      const uint32_t kb = ring_base + st * L::kStage;
      if (ntok > 0) {
        const uint32_t vb = kb + L::kKTile;
        if (!PIPE) scores(kb, s_cur);
        const float (&s)[NT][4] = s_cur;
        // online softmax over the tile's tokens (rows g and g + 8 of this lane)
        const bool v0 = g < ntok, v1 = g + 8 < ntok;
        uint32_t pb[NT][2], pl[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float s0 = v0 ? s[nt][0] * p.scale_log2 : -INFINITY;
          const float s1 = v0 ? s[nt][1] * p.scale_log2 : -INFINITY;
          const float s2 = v1 ? s[nt][2] * p.scale_log2 : -INFINITY;
          const float s3 = v1 ? s[nt][3] * p.scale_log2 : -INFINITY;
          float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
          const float al0 = exp2f(m[nt][0] - mn0), al1 = exp2f(m[nt][1] - mn1);
          m[nt][0] = mn0;
          m[nt][1] = mn1;
          const float p0 = exp2f(s0 - mn0), p1 = exp2f(s1 - mn1);
          const float p2 = exp2f(s2 - mn0), p3 = exp2f(s3 - mn1);
          l[nt][0] = l[nt][0] * al0 + (p0 + p2);
          l[nt][1] = l[nt][1] * al1 + (p1 + p3);
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            o[mt][nt][0] *= al0;
            o[mt][nt][1] *= al1;
            o[mt][nt][2] *= al0;
            o[mt][nt][3] *= al1;
          }
          // P enters the MMA as a 16-bit hi + lo pair so that the weights keep
          // ~16 bits: one rounded copy alone would bias the value mix against
          // the fp32 row sum l by up to 2^-9 relative.
          uint32_t h01, l01, h23, l23;
          split2<CT>(p0, p1, h01, l01);
          split2<CT>(p2, p3, h23, l23);
          pb[nt][0] = movmatrix_trans(h01);
          pb[nt][1] = movmatrix_trans(h23);
          pl[nt][0] = movmatrix_trans(l01);
          pl[nt][1] = movmatrix_trans(l23);
        }
        // zero the V^T fragment entries of tokens past the end (stale ring contents);
        // a full tile skips the masking (the value MMA below, instantiated twice)
        const int tk = 2 * tq;
        const uint32_t mlo = (tk < ntok ? 0x0000ffffu : 0u) | (tk + 1 < ntok ? 0xffff0000u : 0u);
        const uint32_t mhi = (tk + 8 < ntok ? 0x0000ffffu : 0u) | (tk + 9 < ntok ? 0xffff0000u : 0u);
        auto value_mma = [&](auto ragged) {
          constexpr bool RAGGED = decltype(ragged)::value;
          // O^T (D x 8NT) += V^T P
          if (KV8) {
            // a transposed ldmatrix block (8 tokens x 16 codes read as 8 x 8 pairs)
            // gives lane (g, tq) the codes of dims 16 c + 2g, 16 c + 2g + 1 for tokens
            // t0 + 2tq, t0 + 2tq + 1; one byte permute pairs them per dim.  So m-tile
            // c's fragment rows g and g + 8 are dims 16 c + 2g and 16 c + 2g + 1
            // (the epilogue writes them there).
#pragma unroll
            for (int x = 0; x < KS / 2; ++x) {
              uint32_t r[4];
              ldsm_x4_trans(x8_addr(vb, x), r);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int mt = 2 * x + h;
                uint32_t a[4];
                e4m3x4_to_f16x2(__byte_perm(r[2 * h], 0u, 0x3120u), a[0], a[1]);      // tokens 2tq..
                e4m3x4_to_f16x2(__byte_perm(r[2 * h + 1], 0u, 0x3120u), a[2], a[3]);  // 2tq + 8..
                if (RAGGED) {
                  a[0] &= mlo;
                  a[1] &= mlo;
                  a[2] &= mhi;
                  a[3] &= mhi;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  mma_16816<CT>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
                  mma_16816<CT>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
                }
              }
            }
          } else {
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              uint32_t a[4];
              ldsm_x4_trans(vb + sw128_offset(v_row, mt * 16 + v_col, kTile), a);
              if (RAGGED) {
                a[0] &= mlo;
                a[1] &= mlo;
                a[2] &= mhi;
                a[3] &= mhi;
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_16816<CT>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
                mma_16816<CT>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
              }
            }
          }
        };
        if (ntok < kTile) value_mma(std::true_type{});
        else value_mma(std::false_type{});
      }
      __syncwarp();              // every lane is done with this stage
      if (!aborted) issue_next();
      if (PIPE) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) s_cur[nt][e] = s_nxt[nt][e];
        ok_cur = ok_nxt;
      }
    }

    // ---- finish the segment (or this warp's piece of it)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l[nt][e];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        l[nt][e] = v;
      }
    const long long seg = static_cast<long long>(b) * p.Hkv + kvh;
    const long long slot = gw + seg;
    uint16_t *orow = reinterpret_cast<uint16_t *>(p.out) +
                     (static_cast<long long>(b) * p.Hq + kvh * p.G) * D;
    if (has_tiles) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = nt * 8 + 2 * tq + e;
          if (h >= p.G) continue;
          const float inv = l[nt][e] > 0.f ? p.v_scale / l[nt][e] : 0.f;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int d = KV8 ? mt * 16 + 2 * g + hf : mt * 16 + g + hf * 8;
              const float val = o[mt][nt][hf * 2 + e] * inv;
              if (whole) orow[h * D + d] = to16<BF16>(val);
              else p.part_o[(slot * p.G + h) * D + d] = val;
            }
          if (!whole && g == 0)
            p.part_lse[slot * p.G + h] = l[nt][e] > 0.f ? m[nt][e] + log2f(l[nt][e]) : -INFINITY;
        }
    }
    // single-pass merge: only a piece's first and last segments can be split;
    // their arrivals wait until the piece is done, off the streaming path
    if (FUSED && !whole && has_tiles && n_split < 2) {
      split_seg[n_split] = seg;
      split_first[n_split] = tile_first;
      split_tiles[n_split] = P;
      ++n_split;
    }
    // advance to the next segment
    b = nb_;
    kvh = nkvh;
    ctx = nctx;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qf[nt][ks][0] = nq[nt][ks][0];
        qf[nt][ks][1] = nq[nt][ks][1];
      }
  }

  // An aborted piece (a wait timed out) still counts itself in, so that every
  // counter it shares returns to zero and a replayed graph, which reuses the
  // epoch, starts from a clean count; the segment is then merged only if the
  // last arrival is a piece that completed (the output is invalid either way and
  // the status word says so).
  if (FUSED && n_split > 0) {
    __threadfence();                     // every lane's partial rows before the arrivals
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (i >= n_split) break;
      const long long sg = split_seg[i];
      const int g0 = piece_of(split_first[i], TP, pieces);
      const int g1 = piece_of(split_first[i] + split_tiles[i] - 1, TP, pieces);
      const int expected = pieces_with_tiles(g0, g1, TP, pieces, lane);
      if (segment_arrive_last(p.seg_ctr + sg, p.epoch, expected, lane) && !aborted) {
        const long long sb = sg / p.Hkv, skv = sg - sb * p.Hkv;
        uint16_t *rows = reinterpret_cast<uint16_t *>(p.out) + (sb * p.Hq + skv * p.G) * D;
        merge_segment_warp<D, 8 * NT, BF16>(p.part_o, p.part_lse, sg, p.G, g0, g1, TP, pieces,
                                           rows, lane);
      }
    }
  }

  if (aborted && lane == 0) {
    // leave no copy in flight into shared memory: wait (bounded) for the last R tiles
    volatile int never = 0;
    for (long long x = issued > wb + R ? issued - R : wb; x < issued; ++x) {
      const long long n = x - wb;
      mbar_wait(&full[n % R], static_cast<uint32_t>((n / R) & 1), &never);
    }
  }
}

}  // namespace pa
