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
// grid drains and wait on griddepcontrol before reading its results.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct MergeParams {
  const float *part_o;       // [slots][G][DV]
  const float *part_lse;     // [slots][G]
  const int32_t *prefix;     // [B + 1] tiles per kv head (written by the partition pass)
  void *out;                 // [B][Hq][DV] 16-bit
  int B, Hq, Hkv, G;
  int pieces;                // pieces launched by the partition pass
  int min_tiles;             // the partition pass's min_tiles and floor of pieces
  long long floor_pieces;    // (see used_pieces)
};

constexpr int kMergeThreads = 256;

template <int DV, bool BF16>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const MergeParams p) {
  constexpr int TPR = DV / 4;                    // threads per partial row (float4 each)
  constexpr int PG = kMergeThreads / TPR;        // piece groups
  static_assert(TPR * PG == kMergeThreads, "DV/4 must divide the block size");
  __shared__ float red[kMergeThreads / 32];
  __shared__ float4 acc_s[PG][TPR];
  __shared__ float w_s[PG];

  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int seg = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int b = seg / p.Hkv, kvh = seg - (seg / p.Hkv) * p.Hkv;
  const int P = p.prefix[b + 1] - p.prefix[b];
  if (P <= 0 || h >= p.G) return;
  const long long TP = static_cast<long long>(p.Hkv) * p.prefix[p.B];
  const int pieces = used_pieces(p.pieces, TP, p.min_tiles, p.floor_pieces);
  const long long first = static_cast<long long>(p.Hkv) * p.prefix[b] + static_cast<long long>(kvh) * P;
  const int g0 = piece_of(first, TP, pieces);
  const int g1 = piece_of(first + P - 1, TP, pieces);
  if (g0 == g1) return;

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
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * kMergeRowsPerCta + (threadIdx.x >> 5);
  const long long segs = static_cast<long long>(p.B) * p.Hkv;
  if (r >= segs * p.G) return;
  const int seg = static_cast<int>(r / p.G), h = static_cast<int>(r - static_cast<long long>(seg) * p.G);
  const int b = seg / p.Hkv, kvh = seg - (seg / p.Hkv) * p.Hkv;
  const int P = p.prefix[b + 1] - p.prefix[b];
  if (P <= 0) return;
  const long long TP = static_cast<long long>(p.Hkv) * p.prefix[p.B];
  const int pieces = used_pieces(p.pieces, TP, p.min_tiles, p.floor_pieces);
  const long long first = static_cast<long long>(p.Hkv) * p.prefix[b] + static_cast<long long>(kvh) * P;
  const int g0 = piece_of(first, TP, pieces);
  const int g1 = piece_of(first + P - 1, TP, pieces);
  if (g0 == g1) return;

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
