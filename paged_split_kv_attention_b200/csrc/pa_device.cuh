// pa_device.cuh -- sm_100a device helpers: mbarriers with bounded waits, TMA
// tensor copies, warp-level tensor-core fragments and small reductions.
//
// Every wait on an mbarrier is bounded: after PA_WAIT_TIMEOUT_NS of wall time
// (or a hard iteration cap) it gives up, and the caller records PA_ERR_TIMEOUT in
// the device status word and leaves its loop instead of spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifndef PA_WAIT_TIMEOUT_NS
#define PA_WAIT_TIMEOUT_NS 1000000000ull   // 1 s
#endif
#define PA_WAIT_MAX_ITERS (1u << 30)

namespace pa {

// Device status word: first error recorded by any kernel (0 = none).
__device__ int g_status;

// Test hook of the timeout path (pa_test_inject_stall): while nonzero, one warp
// of every partition launch waits on a barrier that nothing completes before it
// issues any copy.  Read by the kernels when they run, so a launch captured in a
// CUDA graph sees the value current at replay time.
__device__ int g_stall_test;

__device__ __forceinline__ bool stall_test_enabled() {
  return *reinterpret_cast<volatile int *>(&g_stall_test) != 0;
}

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false when
// the CTA-wide abort flag is raised or the wait ran out of time; in the latter
// case the abort flag is raised and PA_ERR_TIMEOUT recorded.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1; it < PA_WAIT_MAX_ITERS; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > PA_WAIT_TIMEOUT_NS) break;
    }
  }
  *abort_flag = 1;
  record_error(5 /* PA_ERR_TIMEOUT */);
  return false;
}

// ---------------------------------------------------------------- cp.async

// 16-byte asynchronous copy global -> shared (L2 only).
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed; the
// arrival counts toward the barrier's expected count (noinc).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled tensor load into shared memory, completion counted on `bar`.
// x (innermost coordinate, elements) must be a multiple of 8 for 16-bit data.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map,
                                                 uint64_t *bar, int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Prefetch a 2-D tile of a tensor map into L2 (no shared memory, no completion).
// Prefetch `bytes` (a multiple of 16) from a 16-byte aligned global address into
// L2 with a cache policy (no shared memory, no completion).
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes, uint64_t policy) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(p), "r"(bytes),
               "l"(policy)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z,
                                                uint64_t policy) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile.L2::cache_hint [%0, {%1, %2, %3}], %4;"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "l"(policy)
               : "memory");
}

// 3-D tiled tensor load (same completion and cache hint as the 2-D form).
__device__ __forceinline__ void tma_load_3d_hint(void *dst, const CUtensorMap *map,
                                                 uint64_t *bar, int x, int y, int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------- warp MMA fragments

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D(16x8, f32) += A(16x16) * B(16x8), A row-major, B column-major.
template <bool BF16>
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Two floats -> packed 16-bit pair (round to nearest even), low half = first.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
}

// Split two floats into a rounded 16-bit pair `hi` and the rounded remainder
// `lo` (x ~= hi + lo to about 2^-16 relative), each packed low half first.
template <bool BF16>
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  hi = pack2<BF16>(a, b);
  float ah, bh;
  if constexpr (BF16) {
    ah = __uint_as_float(hi << 16);
    bh = __uint_as_float(hi & 0xffff0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
    ah = f.x;
    bh = f.y;
  }
  lo = pack2<BF16>(a - ah, b - bh);
}

template <bool BF16>
__device__ __forceinline__ uint16_t to16(float x) {
  if constexpr (BF16) {
    __nv_bfloat16 v = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&v);
  } else {
    __half v = __float2half_rn(x);
    return *reinterpret_cast<uint16_t *>(&v);
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Byte offset of (row, col) of a 16-bit tile stored by TMA with 128-byte
// swizzling in 64-column slabs of `rows` rows each (slab = rows x 128 B).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows) {
  return static_cast<uint32_t>((col >> 6) * rows * 128 + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4) + ((col & 7) << 1));
}

__host__ __device__ __forceinline__ int clamp_ctx(int c, int cap) { return c < 0 ? 0 : (c > cap ? cap : c); }

// Work units of a sequence of c tokens: its tiles, plus `extra` units standing
// for the fixed cost of a segment (none for an empty sequence).
__host__ __device__ __forceinline__ int seq_units(int c, int cap, int tile, int extra) {
  const int P = (clamp_ctx(c, cap) + tile - 1) / tile;
  return P > 0 ? P + extra : 0;
}

// prefix[0] = 0, prefix[b + 1] = sum_{b' <= b} seq_units(ctx[b']).  All threads.
template <int NTHREADS>
__device__ void tiles_prefix(const int32_t *ctx, int B, int cap, int tile, int *prefix,
                             int *scratch, bool report, int extra = 0) {
  const int per = (B + NTHREADS - 1) / NTHREADS;
  const int b0 = threadIdx.x * per;
  const int b1 = min(B, b0 + per);
  int local = 0;
  for (int b = b0; b < b1; ++b) {
    const int c = ctx[b];
    if (report && (c < 0 || c > cap)) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
    local += seq_units(c, cap, tile, extra);
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
    run += seq_units(ctx[b], cap, tile, extra);
    prefix[b + 1] = run;
  }
  __syncthreads();
}

// Partition of a flattened work stream of `total` units into `parts` equal
// pieces: piece c covers [begin(c), begin(c + 1)).
__host__ __device__ __forceinline__ long long piece_begin(long long c, long long total, long long parts) {
  return (c * total) / parts;
}

// Pieces actually used out of `parts` launched.  With min_units > 0 (an
// automatic launch) a short stream is cut into the fewest pieces of at most
// min_units units each (so pieces stay near min_units and the partial outputs
// and their merge stay small next to the work itself), but into at least
// floor_pieces pieces, so that a short stream still spreads over several warps;
// with min_units == 0 (an explicit partition count) every piece is used.  The
// partition and merge kernels compute it from the same arguments.
__host__ __device__ __forceinline__ int used_pieces(int parts, long long total, int min_units,
                                           long long floor_pieces) {
  if (min_units <= 0) return parts;
  long long want = (total + min_units - 1) / min_units;
  if (want < floor_pieces) want = floor_pieces;
  return static_cast<int>(want < 1 ? 1 : (want < parts ? want : parts));
}

// The piece that owns unit t (0 <= t < total).
__host__ __device__ __forceinline__ int piece_of(long long t, long long total, long long parts) {
  return static_cast<int>(((t + 1) * parts + total - 1) / total - 1);
}

}  // namespace pa
