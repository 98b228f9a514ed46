// pa_gqa.cuh -- partition pass of paged split-KV decode for grouped query heads.
//
// What it computes (page "cidian.kuaisou.com: flash decoding ++", snippets on the
// three Flash-Decoding steps): the KV stream of every (sequence, kv head) is cut
// into pieces along the sequence; for each piece and each of the G query heads
// that share the kv head, attention over the piece's tokens is computed with a
// running max and sum, and the piece's normalised output plus the log-sum-exp of
// its softmax row are recorded for the merge pass.  A piece that covers a whole
// (sequence, kv head) writes the final output directly.
//
// How the pieces are chosen.  The KV stream is flattened into 16-token tiles in
// (sequence, kv head, tile) order; grid CTA c owns tiles [c*T/P, (c+1)*T/P) of the
// T tiles, so every CTA reads the same number of bytes whatever the mix of
// context lengths.  Where a CTA's range crosses (sequence, kv head) boundaries it
// produces one partial result per segment it touches (slot c + segment).  The
// split points therefore fall where the work balances, not at a fixed length.
//
// Data movement (the pages ask that K and V be loaded in parallel as fast as
// possible, then rescaled and combined).  Warp 0 is a producer: it walks the
// CTA's tiles, looks up each tile's physical block through the block table and
// issues TMA tensor copies of the 16 x D K and V tiles (128-byte swizzle, L2
// evict-first) into an S-stage shared-memory ring guarded by mbarriers.  Warps
// 1..4 consume tiles round-robin.  Per tile a consumer computes S^T = K Q^T with
// mma.sync m16n8k16 (tokens on M, the group's heads on N), the online softmax in
// registers (max over tokens with three xor shuffles, sums kept per lane), and
// O^T += V^T P with V^T fragments from ldmatrix.trans and P moved to the B
// operand layout with movmatrix (as a 16-bit hi + lo pair, two MMAs).  At the end of each segment the four consumer
// warps combine their (max, sum, O) states through shared memory.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kTile = 16;            // tokens per pipeline tile
constexpr int kConsumerWarps = 4;
constexpr int kGqaThreads = 32 * (1 + kConsumerWarps);

struct GqaParams {
  const int32_t *block_table;   // [B][mbs]
  const int32_t *context_lens;  // [B]
  void *out;                    // [B][Hq][D] 16-bit
  float *part_o;                // [slots][G][D]
  float *part_lse;              // [slots][G], log2 domain
  int32_t *prefix_out;          // [B+1] tiles per kv head, written by CTA 0 for the merge
  int B, Hq, Hkv, G, bs, mbs, nb;
  int tiles_per_block;          // bs / 16
  int parts;                    // gridDim.x
  float scale_log2;             // scale * log2(e)
};

template <int D, int NT, int S>
struct GqaLayout {
  static constexpr int kHeads = 8 * NT;            // group width padded to the MMA N
  static constexpr int kKTile = kTile * D * 2;     // bytes of one K (or V) tile
  static constexpr int kStage = 2 * kKTile;
  static constexpr int kQTile = kHeads * D * 2;
  static constexpr int kCombStride = D + 4;        // floats per head row (bank spread)
  static constexpr int kCombWarp = kHeads * kCombStride * 4 + 2 * kHeads * 4;
  static constexpr int ring = 0;
  static constexpr int qbuf = ring + S * kStage;
  static constexpr int comb = qbuf + 2 * kQTile;
  static constexpr int bars = comb + kConsumerWarps * kCombWarp;
  static constexpr int nbars = 2 * S + 4;
  static constexpr int info = bars + nbars * 8;     // int stage_ntok[S]
  static constexpr int flags = info + S * 4;        // abort flag + scan scratch (16 ints)
  static constexpr int prefix = flags + 64;         // int prefix[B + 1]
  static size_t bytes(int B) { return 1024 + prefix + static_cast<size_t>(B + 1) * 4; }
  static_assert(kStage % 1024 == 0 && kQTile % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(bars % 8 == 0, "mbarriers need 8-byte alignment");
};

__device__ __forceinline__ int clamp_ctx(int c, int cap) { return c < 0 ? 0 : (c > cap ? cap : c); }

// prefix[0] = 0, prefix[b + 1] = sum_{b' <= b} ceil(clamp(ctx[b']) / tile).  All threads.
template <int NTHREADS>
__device__ void tiles_prefix(const int32_t *ctx, int B, int cap, int tile, int *prefix,
                             int *scratch, bool report) {
  const int per = (B + NTHREADS - 1) / NTHREADS;
  const int b0 = threadIdx.x * per;
  const int b1 = min(B, b0 + per);
  int local = 0;
  for (int b = b0; b < b1; ++b) {
    const int c = ctx[b];
    if (report && (c < 0 || c > cap)) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
    local += (clamp_ctx(c, cap) + tile - 1) / tile;
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) scratch[w] = v;
  __syncthreads();
  int run = v - local;
  for (int i = 0; i < w; ++i) run += scratch[i];
  if (threadIdx.x == 0) prefix[0] = 0;
  for (int b = b0; b < b1; ++b) {
    run += (clamp_ctx(ctx[b], cap) + tile - 1) / tile;
    prefix[b + 1] = run;
  }
  __syncthreads();
}

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

template <int D, int NT, bool BF16, int S>
__global__ void __launch_bounds__(kGqaThreads, 1)
gqa_partition_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const GqaParams p) {
  using L = GqaLayout<D, NT, S>;
  static_assert(S % kConsumerWarps == 0, "each consumer warp owns fixed ring stages");
  constexpr int KS = D / 16;                 // k-steps of the score MMA / m-tiles of the PV MMA

  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::bars);
  uint64_t *empty = full + S;
  uint64_t *qfull = empty + S;
  uint64_t *qempty = qfull + 2;
  int *stage_ntok = reinterpret_cast<int *>(sm + L::info);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::flags);
  int *scan_scratch = reinterpret_cast<int *>(sm + L::flags) + 4;
  int *prefix = reinterpret_cast<int *>(sm + L::prefix);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int cap = p.mbs * p.bs;

  tiles_prefix<kGqaThreads>(p.context_lens, p.B, cap, kTile, prefix, scan_scratch, c == 0);
  if (c == 0)
    for (int i = tid; i <= p.B; i += kGqaThreads) p.prefix_out[i] = prefix[i];

  const long long TP = static_cast<long long>(p.Hkv) * prefix[p.B];
  const long long t_begin = piece_begin(c, TP, p.parts);
  const long long t_end = piece_begin(c + 1, TP, p.parts);
  if (t_begin >= t_end) return;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const uint64_t policy = l2_evict_first_policy();
    long long issued = 0;     // tiles issued (lane 0)
    int q_issued = 0;         // query tiles issued (lane 0)
    int seg_k = -1;           // segment ordinal in this CTA (lane 0)
    bool aborted = false;
    for (long long base = t_begin; base < t_end && !aborted; base += 32) {
      const long long t = base + lane;
      int b = 0, kvh = 0, j = 0, ntok = 0, row = 0, seg_start = 0;
      if (t < t_end) {
        locate_tile(prefix, p.B, p.Hkv, t, b, kvh, j);
        const int ctx = clamp_ctx(p.context_lens[b], cap);
        ntok = min(kTile, ctx - j * kTile);
        const int jb = j / p.tiles_per_block;
        const int blk = p.block_table[static_cast<long long>(b) * p.mbs + jb];
        if (blk < 0 || blk >= p.nb) {
          record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
          ntok = 0;
        } else {
          row = (blk * p.Hkv + kvh) * p.bs + (j - jb * p.tiles_per_block) * kTile;
        }
        seg_start = (j == 0 || t == t_begin) ? 1 : 0;
      }
      const int n = static_cast<int>(min(32ll, t_end - base));
      for (int i = 0; i < n; ++i) {
        const int bi = __shfl_sync(0xffffffffu, b, i);
        const int kvi = __shfl_sync(0xffffffffu, kvh, i);
        const int ni = __shfl_sync(0xffffffffu, ntok, i);
        const int ri = __shfl_sync(0xffffffffu, row, i);
        const int si = __shfl_sync(0xffffffffu, seg_start, i);
        if (lane == 0 && !aborted) {
          if (si) {
            ++seg_k;
            const int qs = seg_k & 1;
            if (!mbar_wait(&qempty[qs], ((seg_k >> 1) & 1) ^ 1, abort_flag)) {
              aborted = true;
            } else {
              mbar_arrive_expect_tx(&qfull[qs], L::kQTile);
              uint8_t *qdst = sm + L::qbuf + qs * L::kQTile;
#pragma unroll
              for (int x = 0; x < D; x += 64)
                tma_load_2d(qdst + (x / 64) * L::kHeads * 128, &tm_q, &qfull[qs], x,
                            bi * p.Hq + kvi * p.G);
              q_issued = seg_k + 1;
            }
          }
          const long long li = base + i - t_begin;
          const int st = static_cast<int>(li % S);
          const uint32_t ph = static_cast<uint32_t>((li / S) & 1);
          if (!aborted && !mbar_wait(&empty[st], ph ^ 1, abort_flag)) aborted = true;
          if (!aborted) {
            stage_ntok[st] = ni;
            if (ni > 0) {
              mbar_arrive_expect_tx(&full[st], L::kStage);
              uint8_t *kdst = sm + L::ring + st * L::kStage;
#pragma unroll
              for (int x = 0; x < D; x += 64) {
                tma_load_2d_hint(kdst + (x / 64) * kTile * 128, &tm_k, &full[st], x, ri, policy);
                tma_load_2d_hint(kdst + L::kKTile + (x / 64) * kTile * 128, &tm_v, &full[st], x,
                                 ri, policy);
              }
            } else {
              mbar_arrive(&full[st]);
            }
            issued = li + 1;
          }
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && aborted) {
      // Leave no copy in flight into this CTA's shared memory: wait (bounded) for
      // the most recent S tiles and the last two Q tiles to land.
      volatile int never = 0;
      for (long long li = issued > S ? issued - S : 0; li < issued; ++li)
        mbar_wait(&full[li % S], static_cast<uint32_t>((li / S) & 1), &never);
      for (int k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
        mbar_wait(&qfull[k & 1], static_cast<uint32_t>((k >> 1) & 1), &never);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int g = lane >> 2;          // fragment row group
  const int tq = lane & 3;          // thread in quad
  float *comb_all = reinterpret_cast<float *>(sm + L::comb);
  float *comb_me = comb_all + cw * (L::kCombWarp / 4);
  const uint32_t ring_base = smem_u32(sm + L::ring);
  const uint32_t q_base = smem_u32(sm + L::qbuf);
  // per-lane ldmatrix row/column offsets (see fragment layouts in the header comment)
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8, k_col = (lane >> 4) * 8;
  const int v_row = (lane & 7) + (lane >> 4) * 8, v_col = ((lane >> 3) & 1) * 8;
  const int q_row = lane & 7, q_col = (lane >> 3) * 8;

  long long t = t_begin;
  int seg_k = -1;
  while (t < t_end) {
    ++seg_k;
    int b, kvh, j0;
    locate_tile(prefix, p.B, p.Hkv, t, b, kvh, j0);
    const int P = prefix[b + 1] - prefix[b];
    const long long seg_first = static_cast<long long>(p.Hkv) * prefix[b] +
                                static_cast<long long>(kvh) * P;
    const long long seg_end = min(t_end, seg_first + P);
    const bool whole = seg_first >= t_begin && seg_first + P <= t_end;

    // query fragments of this group: B operand (Q^T, d x heads), two k-steps per ldmatrix.x4
    uint32_t qf[NT][KS][2];
    const int qs = seg_k & 1;
    // every lane waits (acquire), then the warp agrees so that collective
    // instructions below run converged even if a wait gave up on some lane
    const bool qok = __all_sync(0xffffffffu, mbar_wait(&qfull[qs], (seg_k >> 1) & 1, abort_flag));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int ks = 0; ks < KS; ks += 2) {
        uint32_t r[4];
        ldsm_x4(q_base + qs * L::kQTile + sw128_offset(nt * 8 + q_row, ks * 16 + q_col, L::kHeads),
                r);
        qf[nt][ks][0] = r[0];
        qf[nt][ks][1] = r[1];
        qf[nt][ks + 1][0] = r[2];
        qf[nt][ks + 1][1] = r[3];
      }
    __syncwarp();
    if (lane == 0 && qok) mbar_arrive(&qempty[qs]);

    float m[NT][2], l[NT][2], o[KS][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    }

    const long long li_first = t - t_begin;
    const long long li_end = seg_end - t_begin;
    long long li = li_first + ((cw - static_cast<int>(li_first % kConsumerWarps)) + kConsumerWarps) %
                                  kConsumerWarps;
    for (; li < li_end; li += kConsumerWarps) {
      const int st = static_cast<int>(li % S);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&full[st], static_cast<uint32_t>((li / S) & 1), abort_flag)))
        continue;
      const int ntok = stage_ntok[st];
      if (ntok > 0) {
        const uint32_t kb = ring_base + st * L::kStage;
        const uint32_t vb = kb + L::kKTile;
        // S^T (16 tokens x 8NT heads) = K Q^T
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a[4];
          ldsm_x4(kb + sw128_offset(k_row, ks * 16 + k_col, kTile), a);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816<BF16>(s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
        }
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
          split2<BF16>(p0, p1, h01, l01);
          split2<BF16>(p2, p3, h23, l23);
          pb[nt][0] = movmatrix_trans(h01);
          pb[nt][1] = movmatrix_trans(h23);
          pl[nt][0] = movmatrix_trans(l01);
          pl[nt][1] = movmatrix_trans(l23);
        }
        // zero the V^T fragment entries of tokens past the end (stale ring contents)
        const int tk = 2 * tq;
        const uint32_t mlo = (tk < ntok ? 0x0000ffffu : 0u) | (tk + 1 < ntok ? 0xffff0000u : 0u);
        const uint32_t mhi = (tk + 8 < ntok ? 0x0000ffffu : 0u) | (tk + 9 < ntok ? 0xffff0000u : 0u);
        // O^T (D x 8NT) += V^T P
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          uint32_t a[4];
          ldsm_x4_trans(vb + sw128_offset(v_row, mt * 16 + v_col, kTile), a);
          a[0] &= mlo;
          a[1] &= mlo;
          a[2] &= mhi;
          a[3] &= mhi;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816<BF16>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
            mma_16816<BF16>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- combine the four consumer warps' states for this segment
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l[nt][e];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        l[nt][e] = v;
      }
    float *cm = comb_me + L::kHeads * L::kCombStride;   // m[kHeads], then l[kHeads]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * tq;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int d0 = mt * 16 + g;
        comb_me[h0 * L::kCombStride + d0] = o[mt][nt][0];
        comb_me[(h0 + 1) * L::kCombStride + d0] = o[mt][nt][1];
        comb_me[h0 * L::kCombStride + d0 + 8] = o[mt][nt][2];
        comb_me[(h0 + 1) * L::kCombStride + d0 + 8] = o[mt][nt][3];
      }
      if (g == 0) {
        cm[h0] = m[nt][0];
        cm[h0 + 1] = m[nt][1];
        cm[L::kHeads + h0] = l[nt][0];
        cm[L::kHeads + h0 + 1] = l[nt][1];
      }
    }
    named_bar_sync(1, 32 * kConsumerWarps);
    {
      const int ct = tid - 32;
      const long long slot = static_cast<long long>(c) + static_cast<long long>(b) * p.Hkv + kvh;
      for (int idx = ct; idx < p.G * D; idx += 32 * kConsumerWarps) {
        const int h = idx / D, d = idx - (idx / D) * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
          M = fmaxf(M, comb_all[w * (L::kCombWarp / 4) + L::kHeads * L::kCombStride + h]);
        float acc = 0.f, Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float *cw_base = comb_all + w * (L::kCombWarp / 4);
          const float mw = cw_base[L::kHeads * L::kCombStride + h];
          const float a = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
          acc += a * cw_base[h * L::kCombStride + d];
          Ls += a * cw_base[L::kHeads * L::kCombStride + L::kHeads + h];
        }
        const float val = Ls > 0.f ? acc / Ls : 0.f;
        if (whole) {
          reinterpret_cast<uint16_t *>(p.out)[(static_cast<long long>(b) * p.Hq + kvh * p.G + h) * D + d] =
              to16<BF16>(val);
        } else {
          p.part_o[(slot * p.G + h) * D + d] = val;
          if (d == 0) p.part_lse[slot * p.G + h] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
        }
      }
    }
    named_bar_sync(1, 32 * kConsumerWarps);
    t = seg_end;
  }
}

}  // namespace pa
