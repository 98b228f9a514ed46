// pa_merge.cuh -- LSE merge pass of paged split-KV decode.
//
// Third Flash-Decoding step (page "cidian.kuaisou.com: flash decoding ++",
// snippets on reducing the per-block outputs and on rescaling and combining
// them; the partial softmax results are brought together once, at the end).
// For one (segment = sequence x kv head, query head h) whose tiles were split
// over pieces pc = g0..g1 of the partition pass, with normalised partial rows
// o_pc and log-sum-exps lse_pc (log2 units) in slot pc + segment:
//
//   M   = max_pc lse_pc
//   w   = 2^(lse_pc - M)
//   out = sum_pc w o_pc / sum_pc w          rounded once to the output type
//
// One CTA per (segment, head) with every partial load of the CTA in flight at
// once: the CTA's threads form PG groups of D/4 threads, group k takes pieces
// g0 + k, g0 + k + PG, ..., each thread one float4 of the row; the groups'
// sums meet in shared memory.  Segments covered by a single piece were written
// by the partition pass and are skipped.  The kernel is launched with
// programmatic dependent launch: its CTAs may be scheduled while the partition
// grid drains.  Each CTA first derives the tile prefix (and so which pieces
// cover its rows) from the sequence lengths, an input, then waits on
// griddepcontrol before reading the partition pass's results.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct MergeParams {
  const float *part_o;       // [slots][G][DV]
  const float *part_lse;     // [slots][G]
  const int32_t *lens;       // [B] the partition pass's sequence lengths (tokens)
  int cap, tile;             // its length clamp and tokens per tile
  int seg_units;             // leading units of a segment that hold no tile
  void *out;                 // [B][Hq][DV] 16-bit
  int B, Hq, Hkv, G;
  int pieces;                // pieces launched by the partition pass
  int min_tiles;             // the partition pass's min_tiles and floor of pieces
  long long floor_pieces;    // (see used_pieces)
};

constexpr int kMergeThreads = 256;

// Dynamic shared memory of a merge CTA: the tile prefix [B + 1] and scan scratch.
__host__ __device__ constexpr size_t merge_smem_bytes(int B) {
  return static_cast<size_t>(B + 1 + 8) * 4;
}

template <int DV, bool BF16>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const MergeParams p) {
  constexpr int TPR = DV / 4;                    // threads per partial row (float4 each)
  constexpr int PG = kMergeThreads / TPR;        // piece groups
  static_assert(TPR * PG == kMergeThreads, "DV/4 must divide the block size");
  __shared__ float red[kMergeThreads / 32];
  __shared__ float4 acc_s[PG][TPR];
  __shared__ float w_s[PG];
  extern __shared__ int merge_prefix[];      // [B + 1], then 8 ints of scan scratch

  tiles_prefix<kMergeThreads>(p.lens, p.B, p.cap, p.tile, merge_prefix,
                              merge_prefix + p.B + 1, false, p.seg_units);
  const int *prefix = merge_prefix;
  const int seg = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int b = seg / p.Hkv, kvh = seg - (seg / p.Hkv) * p.Hkv;
  const int U = prefix[b + 1] - prefix[b];       // the segment's units
  if (U <= 0 || h >= p.G) return;
  const int P = U - p.seg_units;                  // its tiles, after seg_units empty units
  const long long TP = static_cast<long long>(p.Hkv) * prefix[p.B];
  const int pieces = used_pieces(p.pieces, TP, p.min_tiles, p.floor_pieces);
  const long long first = static_cast<long long>(p.Hkv) * prefix[b] +
                          static_cast<long long>(kvh) * U + p.seg_units;
  const int g0 = piece_of(first, TP, pieces);
  const int g1 = piece_of(first + P - 1, TP, pieces);
  if (g0 == g1) return;

  asm volatile("griddepcontrol.wait;" ::: "memory");

  // M = max over the pieces that own tiles (an empty piece wrote nothing)
  float M = -INFINITY;
  for (int pc = g0 + tid; pc <= g1; pc += kMergeThreads)
    if (piece_begin(pc + 1, TP, pieces) > piece_begin(pc, TP, pieces))
      M = fmaxf(M, __ldcg(&p.part_lse[(pc + seg) * p.G + h]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if ((tid & 31) == 0) red[tid >> 5] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int i = 1; i < kMergeThreads / 32; ++i) M = fmaxf(M, red[i]);

  const int pg = tid / TPR, f = tid - (tid / TPR) * TPR;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
#pragma unroll 4
  for (int pc = g0 + pg; pc <= g1; pc += PG) {
    if (piece_begin(pc + 1, TP, pieces) == piece_begin(pc, TP, pieces)) continue;
    const long long row = (pc + seg) * p.G + h;
    const float w = exp2f(__ldcg(&p.part_lse[row]) - M);
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.part_o + row * DV) + f);
    W += w;
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  acc_s[pg][f] = acc;
  if (f == 0) w_s[pg] = W;
  __syncthreads();
  if (pg != 0) return;
#pragma unroll
  for (int k = 1; k < PG; ++k) {
    const float4 v = acc_s[k][f];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
    W += w_s[k];
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                (static_cast<long long>(b) * p.Hq + kvh * p.G + h) * DV + f * 4;
  *reinterpret_cast<uint2 *>(o) = make_uint2(pack2<BF16>(acc.x * inv, acc.y * inv),
                                             pack2<BF16>(acc.z * inv, acc.w * inv));
}

}  // namespace pa

namespace pa {

// Warp-per-row form of the same merge: warp w of a CTA merges flattened row
// r = 8 blockIdx.x + w = segment * G + h.  Lane i fetches the log-sum-exps of
// pieces g0 + i, g0 + i + 32, ... (one round trip for up to 32 pieces), the warp
// takes their max, then every lane accumulates float4 columns i, i + 32, ... of
// the weighted partial rows, four pieces per round so that their loads are in
// flight together.  No block-level barrier: a CTA's rows finish independently.
constexpr int kMergeRowsPerCta = 8;

template <int DV, bool BF16>
__global__ void __launch_bounds__(kMergeRowsPerCta * 32)
merge_rows_kernel(const MergeParams p) {
  constexpr int V4 = DV / 128;                   // float4 columns per lane
  static_assert(V4 * 128 == DV, "DV must be a multiple of 128");
  extern __shared__ int merge_prefix[];          // [B + 1], then 8 ints of scan scratch
  tiles_prefix<kMergeRowsPerCta * 32>(p.lens, p.B, p.cap, p.tile, merge_prefix,
                                      merge_prefix + p.B + 1, false, p.seg_units);
  const int *prefix = merge_prefix;
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * kMergeRowsPerCta + (threadIdx.x >> 5);
  const long long segs = static_cast<long long>(p.B) * p.Hkv;
  if (r >= segs * p.G) return;
  const int seg = static_cast<int>(r / p.G), h = static_cast<int>(r - static_cast<long long>(seg) * p.G);
  const int b = seg / p.Hkv, kvh = seg - (seg / p.Hkv) * p.Hkv;
  const int U = prefix[b + 1] - prefix[b];       // the segment's units
  if (U <= 0) return;
  const int P = U - p.seg_units;                  // its tiles, after seg_units empty units
  const long long TP = static_cast<long long>(p.Hkv) * prefix[p.B];
  const int pieces = used_pieces(p.pieces, TP, p.min_tiles, p.floor_pieces);
  const long long first = static_cast<long long>(p.Hkv) * prefix[b] +
                          static_cast<long long>(kvh) * U + p.seg_units;
  const int g0 = piece_of(first, TP, pieces);
  const int g1 = piece_of(first + P - 1, TP, pieces);
  if (g0 == g1) return;
  // which of the first 32 pieces own tiles (an empty piece wrote nothing)
  const bool own_l = g0 + lane <= g1 &&
                     piece_begin(g0 + lane + 1, TP, pieces) > piece_begin(g0 + lane, TP, pieces);
  const unsigned own = __ballot_sync(0xffffffffu, own_l);

  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Few pieces: the log-sum-exps and every partial row are loaded in one round
  // trip.  Empty pieces enter with weight 0 and a zero row, which leaves the
  // sums exactly as the general loop below forms them.
  constexpr int kFew = DV <= 128 ? 8 : 4;
  if (g1 - g0 < kFew) {
    const float l = own_l ? __ldcg(&p.part_lse[(static_cast<long long>(g0) + lane + seg) * p.G + h])
                          : -INFINITY;
    float4 v[kFew][V4];
#pragma unroll
    for (int i = 0; i < kFew; ++i) {
      const bool e = (own >> i) & 1u;
      const float4 *row = reinterpret_cast<const float4 *>(
          p.part_o + ((static_cast<long long>(g0) + i + seg) * p.G + h) * DV);
#pragma unroll
      for (int k = 0; k < V4; ++k)
        v[i][k] = e ? __ldcg(row + lane + 32 * k) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wl = own_l ? exp2f(l - M) : 0.f;
    float4 acc[V4];
#pragma unroll
    for (int k = 0; k < V4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
#pragma unroll
    for (int i = 0; i < kFew; ++i) {
      const float w = __shfl_sync(0xffffffffu, wl, i);
      W += w;
#pragma unroll
      for (int k = 0; k < V4; ++k) {
        acc[k].x += w * v[i][k].x;
        acc[k].y += w * v[i][k].y;
        acc[k].z += w * v[i][k].z;
        acc[k].w += w * v[i][k].w;
      }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                  (static_cast<long long>(b) * p.Hq + kvh * p.G + h) * DV;
#pragma unroll
    for (int k = 0; k < V4; ++k)
      *reinterpret_cast<uint2 *>(o + 4 * (lane + 32 * k)) =
          make_uint2(pack2<BF16>(acc[k].x * inv, acc[k].y * inv),
                     pack2<BF16>(acc[k].z * inv, acc[k].w * inv));
    return;
  }

  // lse of the pieces that own tiles (an empty piece wrote nothing): -inf else
  auto lse_of = [&](int pc) {
    if (pc > g1 || piece_begin(pc + 1, TP, pieces) == piece_begin(pc, TP, pieces))
      return -INFINITY;
    return __ldcg(&p.part_lse[(static_cast<long long>(pc) + seg) * p.G + h]);
  };
  float l0 = lse_of(g0 + lane);
  float M = l0;
  for (int pc = g0 + 32 + lane; pc <= g1; pc += 32) M = fmaxf(M, lse_of(pc));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float4 acc[V4];
#pragma unroll
  for (int k = 0; k < V4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
  for (int base = g0; base <= g1; base += 32) {
    const float lb = base == g0 ? l0 : lse_of(base + lane);
    const float wl = lb == -INFINITY ? 0.f : exp2f(lb - M);
    const int n = min(32, g1 - base + 1);
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
      const float w = __shfl_sync(0xffffffffu, wl, i);
      if (w == 0.f) continue;                      // empty piece (uniform across the warp)
      const float4 *row = reinterpret_cast<const float4 *>(
          p.part_o + ((static_cast<long long>(base + i) + seg) * p.G + h) * DV);
      W += w;
#pragma unroll
      for (int k = 0; k < V4; ++k) {
        const float4 v = __ldcg(row + lane + 32 * k);
        acc[k].x += w * v.x;
        acc[k].y += w * v.y;
        acc[k].z += w * v.z;
        acc[k].w += w * v.w;
      }
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  uint16_t *o = reinterpret_cast<uint16_t *>(p.out) +
                (static_cast<long long>(b) * p.Hq + kvh * p.G + h) * DV;
#pragma unroll
  for (int k = 0; k < V4; ++k)
    *reinterpret_cast<uint2 *>(o + 4 * (lane + 32 * k)) =
        make_uint2(pack2<BF16>(acc[k].x * inv, acc[k].y * inv),
                   pack2<BF16>(acc[k].z * inv, acc[k].w * inv));
}

}  // namespace pa

namespace pa {

// ---------------------------------------------------------------- fused merge
//
// Single-pass form (the partition kernel merges, no second launch): every piece
// of a split segment, after writing its partial rows, arrives at the segment's
// counter in the workspace; the last of the segment's pieces to arrive merges
// all G rows of the segment with the arithmetic above and writes the output.
//
// A counter is a 64-bit word (call epoch << 32 | arrivals).  A word whose epoch
// is not this call's counts as zero, so a workspace needs no clearing before its
// first call; the last arrival also stores 0, so replays of a captured call
// (same epoch) start from zero too.  The count is taken with compare-and-swap:
// each failed attempt means another piece got in, so the loop ends after at most
// as many rounds as the segment has pieces (bounded besides, as every wait here).

// Lane 0 arrives; the warp learns whether it was the last of `expected`.  The
// caller has fenced its partial rows (every lane) before the first arrival.
__device__ __forceinline__ bool segment_arrive_last(unsigned long long *ctr, uint32_t epoch,
                                                    int expected, int lane) {
  int last = 0;
  if (lane == 0) {
    unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(ctr);
    unsigned long long nw = 0;
    bool done = false;
    for (int it = 0; it < (1 << 20); ++it) {
      const uint32_t cnt = static_cast<uint32_t>(old >> 32) == epoch ? static_cast<uint32_t>(old) : 0u;
      nw = (static_cast<unsigned long long>(epoch) << 32) | (cnt + 1u);
      const unsigned long long got = atomicCAS(ctr, old, nw);
      if (got == old) {
        done = true;
        break;
      }
      old = got;
    }
    if (!done) record_error(5 /* PA_ERR_TIMEOUT */);
    last = done && static_cast<int>(static_cast<uint32_t>(nw)) == expected;
    if (last) *reinterpret_cast<volatile unsigned long long *>(ctr) = 0ull;
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) __threadfence();              // the other pieces' rows after their arrivals
  return last != 0;
}

// Non-empty pieces among g0..g1 (an explicit partition count can exceed the
// tiles, and an empty piece writes nothing).
__device__ __forceinline__ int pieces_with_tiles(int g0, int g1, long long TP, int pieces,
                                                 int lane) {
  int n = 0;
  for (int pc = g0 + lane; pc <= g1; pc += 32)
    n += piece_begin(pc + 1, TP, pieces) > piece_begin(pc, TP, pieces);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
  return n;
}

// One warp merges segment `seg` (pieces g0..g1, G <= GH rows of D) into out_rows
// (the segment's G output rows, 16-bit), eight rows at a time.  Lane l holds the
// weights of piece base + l for the eight rows; float4 i = l + 32k of the rows'
// part of a piece's [G][D] partial block belongs to row i / (D/4) of the eight:
// row k for D = 128, row 2k + l/16 for D = 64.
template <int D, int GH, bool BF16>
__device__ __forceinline__ void merge_segment_warp(const float *part_o, const float *part_lse,
                                                   long long seg, int G, int g0, int g1,
                                                   long long TP, int pieces, uint16_t *out_rows,
                                                   int lane) {
  static_assert(D == 64 || D == 128, "head dims 64 and 128");
  static_assert(GH % 8 == 0, "rows in chunks of eight");
  constexpr int F4 = D / 4;                         // float4 per row
  constexpr int K4 = 8 * F4 / 32;                   // float4 per lane per piece and chunk
  constexpr int kU = 2;                             // pieces whose loads are in flight together
  const int n4 = G * F4;                            // float4 per piece block
  auto lse_at = [&](int pc, int h) {
    return __ldcg(&part_lse[(static_cast<long long>(pc) + seg) * G + h]);
  };
  auto nonempty = [&](int pc) {
    return pc <= g1 && piece_begin(pc + 1, TP, pieces) > piece_begin(pc, TP, pieces);
  };
  // log-sum-exps of the first 32 pieces stay in registers for the weights
  float L0[GH], M[GH];
  const bool mine0 = nonempty(g0 + lane);
#pragma unroll
  for (int h = 0; h < GH; ++h) L0[h] = (mine0 && h < G) ? lse_at(g0 + lane, h) : -INFINITY;
#pragma unroll
  for (int h = 0; h < GH; ++h) M[h] = L0[h];
  for (int pc = g0 + 32 + lane; pc <= g1; pc += 32)
    if (nonempty(pc))
#pragma unroll
      for (int h = 0; h < GH; ++h)
        if (h < G) M[h] = fmaxf(M[h], lse_at(pc, h));
#pragma unroll
  for (int h = 0; h < GH; ++h)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M[h] = fmaxf(M[h], __shfl_xor_sync(0xffffffffu, M[h], off));

#pragma unroll
  for (int hc = 0; hc < GH / 8; ++hc) {
    if (8 * hc >= G) break;
    const int c0 = 8 * hc * F4;                     // first float4 of the chunk's rows
    float4 acc[K4];
#pragma unroll
    for (int k = 0; k < K4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    float W[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) W[j] = 0.f;
    for (int base = g0; base <= g1; base += 32) {
      float wl[8];
      const bool mine = nonempty(base + lane);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int h = 8 * hc + j;
        wl[j] = (mine && h < G)
                    ? exp2f((base == g0 ? L0[h] : lse_at(base + lane, h)) - M[h]) : 0.f;
      }
      const int n = min(32, g1 - base + 1);
      const unsigned ne = __ballot_sync(0xffffffffu, mine);
      // kU pieces per round, their loads issued together; an empty piece (or one
      // past the end) has weight 0 and loads nothing
      for (int i = 0; i < n; i += kU) {
        float4 v[kU][K4];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const bool e = i + u < n && ((ne >> (i + u)) & 1u);
          const float4 *blk = reinterpret_cast<const float4 *>(
              part_o + (static_cast<long long>(base + i + u) + seg) * G * D) + c0;
#pragma unroll
          for (int k = 0; k < K4; ++k)
            v[u][k] = (e && c0 + lane + 32 * k < n4) ? __ldcg(blk + lane + 32 * k)
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int src = (i + u) & 31;
          const bool in = i + u < n;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = __shfl_sync(0xffffffffu, wl[j], src);
            W[j] += in ? x : 0.f;
          }
#pragma unroll
          for (int k = 0; k < K4; ++k) {
            float w;
            if (D == 128) {
              w = __shfl_sync(0xffffffffu, wl[k], src);
            } else {
              const float wa = __shfl_sync(0xffffffffu, wl[2 * k], src);
              const float wb = __shfl_sync(0xffffffffu, wl[2 * k + 1], src);
              w = (lane >> 4) ? wb : wa;
            }
            w = in ? w : 0.f;
            acc[k].x += w * v[u][k].x;
            acc[k].y += w * v[u][k].y;
            acc[k].z += w * v[u][k].z;
            acc[k].w += w * v[u][k].w;
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < K4; ++k) {
      const int i4 = c0 + lane + 32 * k;
      if (i4 >= n4) continue;
      const float Wr = D == 128 ? W[k] : ((lane >> 4) ? W[2 * k + 1] : W[2 * k]);
      const float inv = Wr > 0.f ? 1.f / Wr : 0.f;
      *reinterpret_cast<uint2 *>(out_rows + 4 * i4) =
          make_uint2(pack2<BF16>(acc[k].x * inv, acc[k].y * inv),
                     pack2<BF16>(acc[k].z * inv, acc[k].w * inv));
    }
  }
}

}  // namespace pa
