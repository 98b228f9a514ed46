// pa_merge.cuh -- LSE merge pass of paged split-KV decode.
//
// Third Flash-Decoding step (page "cidian.kuaisou.com: flash decoding ++",
// snippets on reducing the per-block outputs and on rescaling and combining
// them; the partial softmax results are brought together once, at the end).
// For one (sequence, query head) with partial results (o_s, lse_s) from pieces
// s = c0..c1 of the partition pass:
//
//   M   = max_s lse_s
//   w_s = 2^(lse_s - M)                    (lse kept in log2 units)
//   out = sum_s w_s o_s / sum_s w_s        rounded once to the output type
//
// One warp per (sequence, head).  Rows whose segment was covered by a single
// piece were already written by the partition pass and are skipped; rows of
// empty sequences are written as zeros.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct MergeParams {
  const float *part_o;       // [slots][G][DV]
  const float *part_lse;     // [slots][G]
  const int32_t *prefix;     // [B + 1] tiles per kv head (written by the partition pass)
  void *out;                 // [B][Hq][DV] 16-bit
  int B, Hq, Hkv, G;
  int parts;                 // partition-pass grid size
};

constexpr int kMergeWarps = 4;

template <int DV, bool BF16>
__global__ void __launch_bounds__(32 * kMergeWarps)
merge_kernel(const MergeParams p) {
  constexpr int PER = DV / 32;                 // floats per lane
  constexpr int VW = PER >= 4 ? 4 : PER;       // vector width
  constexpr int NV = PER / VW;
  static_assert(PER * 32 == DV && NV * VW == PER, "DV must be a multiple of 32");
  const int lane = threadIdx.x & 31;
  const long long pair = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  if (pair >= static_cast<long long>(p.B) * p.Hq) return;
  const int b = static_cast<int>(pair / p.Hq), h = static_cast<int>(pair % p.Hq);
  const int kvh = h / p.G, g = h - kvh * p.G;
  uint16_t *o = reinterpret_cast<uint16_t *>(p.out) + pair * DV;

  const int P = p.prefix[b + 1] - p.prefix[b];
  if (P <= 0) {
#pragma unroll
    for (int i = 0; i < PER; ++i) o[lane * PER + i] = 0;
    return;
  }
  const long long TP = static_cast<long long>(p.Hkv) * p.prefix[p.B];
  const long long first = static_cast<long long>(p.Hkv) * p.prefix[b] + static_cast<long long>(kvh) * P;
  const int c0 = piece_of(first, TP, p.parts);
  const int c1 = piece_of(first + P - 1, TP, p.parts);
  if (c0 == c1) return;
  const long long seg = static_cast<long long>(b) * p.Hkv + kvh;

  // Pieces with an empty tile range (more pieces than tiles) wrote nothing.
  float M = -INFINITY;
  for (int cc = c0 + lane; cc <= c1; cc += 32)
    if (piece_begin(cc + 1, TP, p.parts) > piece_begin(cc, TP, p.parts))
      M = fmaxf(M, p.part_lse[(cc + seg) * p.G + g]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float W = 0.f;
#pragma unroll 4
  for (int cc = c0; cc <= c1; ++cc) {
    if (piece_begin(cc + 1, TP, p.parts) == piece_begin(cc, TP, p.parts)) continue;
    const long long row = (cc + seg) * p.G + g;
    const float lse = p.part_lse[row];
    const float w = lse == -INFINITY ? 0.f : exp2f(lse - M);
    W += w;
    const float *src = p.part_o + row * DV;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int e = (lane + 32 * v) * VW;
      if constexpr (VW == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(src + e);
        acc[v * 4 + 0] += w * x.x;
        acc[v * 4 + 1] += w * x.y;
        acc[v * 4 + 2] += w * x.z;
        acc[v * 4 + 3] += w * x.w;
      } else if constexpr (VW == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(src + e);
        acc[v * 2 + 0] += w * x.x;
        acc[v * 2 + 1] += w * x.y;
      } else {
        acc[v] += w * src[e];
      }
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int k = 0; k < VW; ++k) o[(lane + 32 * v) * VW + k] = to16<BF16>(acc[v * VW + k] * inv);
}

}  // namespace pa
