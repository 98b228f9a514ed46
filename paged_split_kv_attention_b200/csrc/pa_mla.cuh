// pa_mla.cuh -- MLA (shared-latent) paged split-KV decode: the partition pass on
// the 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes.  All H = 128 query heads of a sequence read one compressed
// latent vector per token (page "wenku.it search: Multi-head Latent Attention
// (MLA)", DeepSeek-V2 abstract on the latent KV): the key is the whole
// 576-wide latent row and the value its first 512 dims, so per sequence
//   out[h, :] = softmax_t(scale * q[h, :] . c_t) c_t[0:512].
// The KV stream is split and merged exactly as for GQA (page
// "cidian.kuaisou.com: flash decoding ++", three-step snippets): the flattened
// stream of 64-token tiles is cut into equal pieces, one per CTA pair; a pair
// that covers a whole sequence writes the output, otherwise it leaves a
// normalised partial and the log-sum-exp of each head row for the merge kernel.
//
// Why a CTA pair.  The value accumulator O (128 heads x 512 fp32) alone fills
// the 512 columns of one SM's tensor memory, so the pair splits the work:
//   CTA r accumulates O[:, 256r : 256r+256]               (256 TMEM columns)
//   CTA r computes the partial score S_r = Q[:, Kr] C[:, Kr]^T over its half of
//   the latent dims, K0 = [0, 320), K1 = [320, 576)        (64 TMEM columns x 2)
// and the two fp32 partial score tiles are exchanged through distributed shared
// memory, so both CTAs hold S = S_0 + S_1 (added in rank order: bit-identical)
// and run the identical softmax.  Each CTA stages latent columns [0, 320) or
// [256, 576) of every tile: its score half plus its value half.
//
// Warp roles (192 threads): warps 0-3 own TMEM lanes 0-127 = head rows (score
// load, exchange, online softmax in log2 units with a lazily raised running max,
// P as a bf16 hi + lo pair into tensor memory, epilogue); warp 4 is the TMA producer (query slabs per
// sequence, latent slabs per tile, block table looked up 32 tiles ahead); warp 5
// issues the MMAs from one thread:
//   S(n) = Q_r . C_r^T    M=128 N=64  K=320|256, A K-major, B K-major (latent)
//   O   += P . V_r        M=128 N=256 K=64 (x2: P hi, P lo), A in TMEM, B MN-major (latent)
// The partial score tiles travel between the pair as bulk copies, 8 KB per warp.
// All operands are TMA-written with the 128-byte swizzle; all waits are bounded.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kMlaTile = 64;              // tokens per tile
constexpr int kMlaHeads = 128;
constexpr int kMlaDk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaStages = 2;
constexpr int kMlaThreads = 192;
constexpr int kMlaRescale = 8;            // raise the running max only past 2^8 growth

struct MlaParams {
  const int32_t *block_table;   // [B][mbs]
  const int32_t *context_lens;  // [B]
  void *out;                    // [B][128][512] bf16
  float *part_o;                // [slots][128][512]
  float *part_lse;              // [slots][128], log2 units
  int32_t *prefix_out;          // [B+1] tiles per sequence (written by CTA 0)
  int B, bs, mbs, nb;
  int tiles_per_block;          // bs / 64
  int parts;                    // CTA pairs (= pieces)
  float scale_log2;
};

struct MlaLayout {
  static constexpr int kQSlab = kMlaHeads * 128;          // 128 rows x 64 bf16
  static constexpr int kLSlab = kMlaTile * 128;           // 64 rows x 64 bf16
  static constexpr int kStage = 5 * kLSlab;               // 40 KB
  static constexpr int q = 0;                             // 5 query slabs
  static constexpr int stage = q + 5 * kQSlab;
  static constexpr int xs = stage + kMlaStages * kStage;  // my partial scores, to send (swizzled)
  static constexpr int x = xs + kMlaHeads * 256;          // partner's partial scores (swizzled)
  static constexpr int bars = x + kMlaHeads * 256;
  static constexpr int nbars = 32;
  static constexpr int misc = bars + nbars * 8;           // tmem base, abort, flags, scan
  static constexpr int info = misc + 64;                  // stage_valid[kMlaStages]
  static constexpr int prefix = info + 16;
  static size_t bytes(int B) { return 1024 + prefix + static_cast<size_t>(B + 1) * 4; }
  static_assert(stage % 1024 == 0 && kStage % 1024 == 0 && xs % 16 == 0, "alignment");
};

// Largest batch whose prefix table still fits next to the buffers above.
constexpr int kMlaMaxBatch = 384;

// ------------------------------------------------------------------ tcgen05 helpers

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t map_remote(uint32_t local_smem, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

__device__ __forceinline__ void remote_arrive(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait with cluster-scope acquire (for barriers the partner CTA arrives on).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1; it < PA_WAIT_MAX_ITERS; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > PA_WAIT_TIMEOUT_NS) break;
    }
  }
  *abort_flag = 1;
  record_error(5 /* PA_ERR_TIMEOUT */);
  return false;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bulk copy of `bytes` from this CTA's shared memory to the partner's, completion
// counted (complete_tx) on the partner's mbarrier; tracked in a bulk async-group.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src_cta,
                                                  uint32_t bytes, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t"
      "cp.async.bulk.commit_group;" ::"r"(dst_cluster),
      "r"(src_cta), "r"(bytes), "r"(bar_cluster)
      : "memory");
}

// Wait until every bulk copy this thread issued has finished reading its source.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Bounded wait for threads off the critical path: back off between probes so
// that a spinning warp does not take issue slots from the softmax warps.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t *bar, uint32_t parity,
                                               volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1; it < PA_WAIT_MAX_ITERS; ++it) {
    __nanosleep(32);
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > PA_WAIT_TIMEOUT_NS) break;
    }
  }
  *abort_flag = 1;
  record_error(5 /* PA_ERR_TIMEOUT */);
  return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory matrix descriptor, 128-byte swizzle (layout type 2, version 1).
__device__ __forceinline__ uint64_t umma_desc(uint32_t smem_addr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF) |
         (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, both K-major unless b_mn.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Same with the A operand (M x K, 16-bit pairs per 32-bit column) in tensor memory.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                                 uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(tmem_d), "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns (one row slice per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ work walk

// Sequence b and tile j of flattened MLA tile t (0 <= t < prefix[B]).
__device__ __forceinline__ void mla_locate(const int *prefix, int B, long long t, int &b, int &j) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  b = lo;
  j = static_cast<int>(t - prefix[b]);
}

__device__ __forceinline__ int mla_tile_row(const MlaParams &p, const int *prefix, long long t) {
  int b, j;
  mla_locate(prefix, p.B, t, b, j);
  const int jb = j / p.tiles_per_block;
  const int blk = __ldg(&p.block_table[static_cast<long long>(b) * p.mbs + jb]);
  if (blk < 0 || blk >= p.nb) return -1;
  return blk * p.bs + (j - jb * p.tiles_per_block) * kMlaTile;
}

// barrier slots
enum MlaBar {
  kLatFull = 0, kLatEmpty = 2, kQFull = 4, kQEmpty = 5, kSFull = 6, kSEmpty = 8, kPFull = 10,
  kPEmpty = 11, kOReady = 12, kOFree = 13, kDone = 14, kFinal = 15,
  kXFull = 16,     // 4 per-warp inboxes: the partner warp's 32 rows landed (tx bytes)
  kXEmpty = 20     // 4 per-warp outboxes: the partner warp has read the rows I sent
};

__global__ void __launch_bounds__(kMlaThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_lat, const MlaParams p) {
  using L = MlaLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::bars);
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(sm + L::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::misc + 4);
  int *scan_scratch = reinterpret_cast<int *>(sm + L::misc + 16);
  int *stage_valid = reinterpret_cast<int *>(sm + L::info);
  int *prefix = reinterpret_cast<int *>(sm + L::prefix);
  float *xbuf = reinterpret_cast<float *>(sm + L::x);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int cap = p.mbs * p.bs;
  // latent columns this CTA stages and the score slabs it contracts over
  const int lat_col0 = rank == 0 ? 0 : 256;
  const int q_col0 = rank == 0 ? 0 : 320;
  const int q_slabs = rank == 0 ? 5 : 4;
  const int s_slab0 = rank == 0 ? 0 : 1;     // first staged latent slab used by the scores

  // ---- prologue (all threads): tiles of 64 tokens per sequence, inclusive prefix
  {
    const int per = (p.B + kMlaThreads - 1) / kMlaThreads;
    const int b0 = tid * per, b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) {
      const int c = p.context_lens[b];
      if (blockIdx.x == 0 && (c < 0 || c > cap)) record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
      local += (min(max(c, 0), cap) + kMlaTile - 1) / kMlaTile;
    }
    int v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) scan_scratch[warp] = v;
    __syncthreads();
    int run = v - local;
    for (int i = 0; i < warp; ++i) run += scan_scratch[i];
    if (tid == 0) prefix[0] = 0;
    for (int b = b0; b < b1; ++b) {
      run += (min(max(p.context_lens[b], 0), cap) + kMlaTile - 1) / kMlaTile;
      prefix[b + 1] = run;
    }
  }
  if (tid == 0) {
    for (int i = 0; i < L::nbars; ++i) {
      uint32_t cnt = 1;
      if (i == kSEmpty || i == kSEmpty + 1 || i == kPFull || i == kOFree) cnt = 4;

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
  // both CTAs' barriers must exist before either arrives remotely
  cluster_sync_all();

  const uint32_t tmem = *tmem_base_s;
  // columns: S buffers 0 and 64, P hi 128, P lo 160, O 256..511
  const uint32_t tm_s0 = tmem, tm_p = tmem + 128, tm_o = tmem + 256;

  if (blockIdx.x == 0)
    for (int i = tid; i <= p.B; i += kMlaThreads) p.prefix_out[i] = prefix[i];
  // empty sequences: all-zero rows (rank 0 of each pair takes a share)
  if (rank == 0)
    for (int b = pair; b < p.B; b += p.parts)
      if (prefix[b + 1] == prefix[b])
        for (int i = tid; i < kMlaHeads * kMlaDv; i += kMlaThreads)
          reinterpret_cast<uint16_t *>(p.out)[static_cast<long long>(b) * kMlaHeads * kMlaDv + i] = 0;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const long long TP = prefix[p.B];
  const long long tb = piece_begin(pair, TP, p.parts), te = piece_begin(pair + 1, TP, p.parts);
  const int ntiles = static_cast<int>(te - tb);

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    const uint64_t policy = l2_evict_first_policy();
    int seg_k = -1, issued = 0, q_issued = 0;
    bool aborted = false;
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_lat);
    }
    for (int base = 0; base < ntiles && !aborted; base += 32) {
      const long long t = tb + base + lane;
      int row = 0, seg_start = 0, b = 0;
      if (base + lane < ntiles) {
        int j;
        mla_locate(prefix, p.B, t, b, j);
        row = mla_tile_row(p, prefix, t);
        seg_start = (j == 0 || base + lane == 0) ? 1 : 0;
      }
      const int n = min(32, ntiles - base);
      for (int i = 0; i < n; ++i) {
        const int ri = __shfl_sync(0xffffffffu, row, i);
        const int si = __shfl_sync(0xffffffffu, seg_start, i);
        const int bi = __shfl_sync(0xffffffffu, b, i);
        if (lane == 0 && !aborted) {
          if (si) {
            ++seg_k;
            if (!mbar_wait_idle(&bar[kQEmpty], (seg_k & 1) ^ 1, abort_flag)) {
              aborted = true;
            } else {
              mbar_arrive_expect_tx(&bar[kQFull], q_slabs * L::kQSlab);
              for (int s = 0; s < q_slabs; ++s)
                tma_load_2d(sm + L::q + s * L::kQSlab, &tm_q, &bar[kQFull], q_col0 + 64 * s,
                            bi * kMlaHeads);
              q_issued = seg_k + 1;
            }
          }
          const int nn = base + i;
          const int st = nn % kMlaStages;
          if (!aborted && !mbar_wait_idle(&bar[kLatEmpty + st], ((nn / kMlaStages) & 1) ^ 1, abort_flag))
            aborted = true;
          if (!aborted) {
            if (ri < 0) {
              record_error(4 /* PA_ERR_BAD_BLOCK_ID */);
              stage_valid[st] = 0;
              mbar_arrive(&bar[kLatFull + st]);
            } else {
              stage_valid[st] = 1;
              mbar_arrive_expect_tx(&bar[kLatFull + st], L::kStage);
              for (int s = 0; s < 5; ++s)
                tma_load_2d_hint(sm + L::stage + st * L::kStage + s * L::kLSlab, &tm_lat,
                                 &bar[kLatFull + st], lat_col0 + 64 * s, ri, policy);
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
      if (q_issued > 0) mbar_wait(&bar[kQFull], (q_issued - 1) & 1, &never);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kMlaTile, false);
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, 256, true);
      const uint32_t q_base = smem_u32(sm + L::q);
      const uint32_t st_base = smem_u32(sm + L::stage);
      bool aborted = false;
      // segment bookkeeping walks the same tiles as the producer
      auto tile_first = [&](int n) {
        int b, j;
        mla_locate(prefix, p.B, tb + n, b, j);
        return n == 0 || j == 0;
      };
      auto tile_last = [&](int n) {
        int b, j;
        mla_locate(prefix, p.B, tb + n, b, j);
        return n == ntiles - 1 || j == prefix[b + 1] - prefix[b] - 1;
      };
      int s_seg = -1;                       // segment ordinal of the last S issued
      auto issue_s = [&](int n) {
        if (aborted) return;
        const int st = n % kMlaStages;
        const bool first = tile_first(n);
        if (first) ++s_seg;
        if (!mbar_wait_idle(&bar[kLatFull + st], (n / kMlaStages) & 1, abort_flag) ||
            (first && !mbar_wait_idle(&bar[kQFull], s_seg & 1, abort_flag)) ||
            !mbar_wait_idle(&bar[kSEmpty + (n & 1)], ((n >> 1) & 1) ^ 1, abort_flag)) {
          aborted = true;
          return;
        }
        tc_fence_after();
        const uint32_t lat = st_base + st * L::kStage;
        const int ksteps = q_slabs * 4;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint64_t a = umma_desc(q_base + (ks >> 2) * L::kQSlab + (ks & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc(lat + (s_slab0 + (ks >> 2)) * L::kLSlab + (ks & 3) * 32, 16,
                                       1024);
          umma_bf16(tm_s0 + (n & 1) * 64, a, b, idesc_s, ks > 0);
        }
        umma_commit(&bar[kSFull + (n & 1)]);
        if (tile_last(n)) umma_commit(&bar[kQEmpty]);
      };
      int o_seg = -1;
      auto issue_pv = [&](int n) {
        if (aborted) return;
        const int st = n % kMlaStages;
        const bool first = tile_first(n);
        if (first) ++o_seg;
        if (!mbar_wait_idle(&bar[kPFull], n & 1, abort_flag) ||
            (first && o_seg > 0 && !mbar_wait_idle(&bar[kOFree], (o_seg - 1) & 1, abort_flag))) {
          aborted = true;
          return;
        }
        tc_fence_after();
        const uint32_t lat = st_base + st * L::kStage;
        for (int kk = 0; kk < kMlaTile / 16; ++kk) {
          const uint64_t b = umma_desc(lat + kk * 2048, L::kLSlab, 1024);
          umma_bf16_tmem_a(tm_o, tm_p + kk * 8, b, idesc_o, !(first && kk == 0));
          umma_bf16_tmem_a(tm_o, tm_p + 32 + kk * 8, b, idesc_o, true);
        }
        umma_commit(&bar[kPEmpty]);
        umma_commit(&bar[kLatEmpty + st]);
        umma_commit(&bar[kOReady]);
      };
      issue_s(0);
      for (int n = 0; n < ntiles && !aborted; ++n) {
        if (tile_last(n)) {
          issue_pv(n);
          if (n + 1 < ntiles) issue_s(n + 1);
        } else {
          if (n + 1 < ntiles) issue_s(n + 1);
          issue_pv(n);
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
    // exchanged row h: 16-byte chunk c at chunk c ^ (h & 15) (conflict-free per quarter warp)
    float *xsend = reinterpret_cast<float *>(sm + L::xs);
    const int xsw = h & 15;
    // this warp's 32 rows (8 KB) travel on their own: warp w of one CTA sends to
    // warp w of the partner, with per-warp inbox / outbox barriers
    const uint32_t rows_off = static_cast<uint32_t>(warp * 32 * 256);
    const uint32_t xrecv_remote = map_remote(smem_u32(xbuf) + rows_off, peer);
    const uint32_t xfull_remote = map_remote(smem_u32(&bar[kXFull + warp]), peer);
    const uint32_t xempty_remote = map_remote(smem_u32(&bar[kXEmpty + warp]), peer);
    bool aborted = false;
    float m_run = -INFINITY, l_run = 0.f;
    int seg_k = -1, b = 0, j = 0, ctx = 0;
    for (int n = 0; n < ntiles; ++n) {
      mla_locate(prefix, p.B, tb + n, b, j);
      const bool first = (n == 0 || j == 0);
      const int P = prefix[b + 1] - prefix[b];
      const bool last = (n == ntiles - 1) || (j == P - 1);
      if (first) {
        ++seg_k;
        m_run = -INFINITY;
        l_run = 0.f;
        ctx = min(max(p.context_lens[b], 0), cap);
      }
      const int ntok = min(kMlaTile, ctx - j * kMlaTile);
      // ---- partial scores of this CTA
      float s[64];
      bool got = !aborted && mbar_wait(&bar[kSFull + (n & 1)], (n >> 1) & 1, abort_flag);
      aborted = !__all_sync(0xffffffffu, got);
      tc_fence_after();
      {
        float v[32];
        tmem_ld32(tm_s0 + (n & 1) * 64 + lane_off, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = v[i];
        tmem_ld32(tm_s0 + (n & 1) * 64 + 32 + lane_off, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 + i] = v[i];
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kSEmpty + (n & 1)]);
      // ---- exchange with the partner: this warp's partial rows go to its slice of
      // the send buffer and leave as one 8 KB bulk copy that completes on the
      // partner warp's inbox; the partner's rows arrive the same way
      if (lane == 0) bulk_wait_read_all();       // the previous send has left the slice
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<float4 *>(xsend + h * 64 + ((c ^ xsw) << 2)) =
            make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && !aborted) {
        mbar_arrive_expect_tx(&bar[kXFull + warp], 32 * 256);
        if (mbar_wait_cluster(&bar[kXEmpty + warp], (n & 1) ^ 1, abort_flag))
          bulk_copy_to_peer(xrecv_remote, smem_u32(xsend) + rows_off, 32 * 256, xfull_remote);
      }
      got = !aborted && mbar_wait_cluster(&bar[kXFull + warp], n & 1, abort_flag);
      aborted = !__all_sync(0xffffffffu, got);
      {
        const float4 *xr = reinterpret_cast<const float4 *>(xbuf + h * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 x4 = xr[i ^ xsw];
          // S = S_0 + S_1 in rank order on both CTAs
          if (rank == 0) {
            s[4 * i] += x4.x; s[4 * i + 1] += x4.y; s[4 * i + 2] += x4.z; s[4 * i + 3] += x4.w;
          } else {
            s[4 * i] = x4.x + s[4 * i]; s[4 * i + 1] = x4.y + s[4 * i + 1];
            s[4 * i + 2] = x4.z + s[4 * i + 2]; s[4 * i + 3] = x4.w + s[4 * i + 3];
          }
        }
      }
      __syncwarp();
      if (!aborted && lane == 0) remote_arrive(xempty_remote);
      // ---- online softmax (log2 units), running max raised lazily
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = i < ntok ? s[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      const bool raise = mt > m_run + kMlaRescale;
      if (__any_sync(0xffffffffu, raise && !first)) {
        // O must be scaled by 2^(m_old - m_new) for the rows whose max moved:
        // wait until the previous tile's value MMA has landed, then rescale in TMEM
        got = !aborted && mbar_wait(&bar[kOReady], (n - 1) & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        const float alpha = (raise && !first) ? ex2_approx(m_run - mt) : 1.f;
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld32(tm_o + c + lane_off, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tm_o + c + lane_off, v);
        }
        tmem_wait_st();
        tc_fence_before();
        if (raise && !first) l_run *= alpha;
      }
      if (raise) m_run = mt;
      // ---- P = 2^(s - m) as a bf16 hi + lo pair (about 16 significant bits: a
      // single bf16 copy would bias the value mix by up to 2^-9 per weight), stored
      // into tensor memory as the A operand of the value MMA
      got = !aborted && mbar_wait(&bar[kPEmpty], (n & 1) ^ 1, abort_flag);
      aborted = !__all_sync(0xffffffffu, got);
      tc_fence_after();
      {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2_approx(s[2 * e] - m_run);
          const float p1 = ex2_approx(s[2 * e + 1] - m_run);
          split2<true>(p0, p1, hi[e], lo[e]);
          l_run += p0 + p1;
        }
        tmem_st32u(tm_p + lane_off, hi);
        tmem_st32u(tm_p + 32 + lane_off, lo);
        tmem_wait_st();
      }
      // tokens past the end: zero their value rows so that 0 x stale data stays 0
      if (ntok < kMlaTile) {
        uint8_t *stg = sm + L::stage + (n % kMlaStages) * L::kStage;
        const int rows = kMlaTile - ntok;
        for (int i = h; i < rows * 4 * 8; i += kMlaHeads) {
          const int slab = i / (rows * 8), r = ntok + (i / 8) % rows, ch = i % 8;
          *reinterpret_cast<uint4 *>(stg + slab * L::kLSlab + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kPFull]);
      // ---- segment end: normalise and write this CTA's half of the rows
      if (last) {
        got = !aborted && mbar_wait(&bar[kOReady], n & 1, abort_flag);
        aborted = !__all_sync(0xffffffffu, got);
        tc_fence_after();
        const long long first_tile = prefix[b];
        const bool whole = first_tile >= tb && first_tile + P <= te;
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const long long slot = pair + b;
        for (int c = 0; c < 256; c += 32) {
          float v[32];
          tmem_ld32(tm_o + c + lane_off, v);
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
              *reinterpret_cast<float4 *>(o + 4 * q4) =
                  make_float4(v[4 * q4] * inv, v[4 * q4 + 1] * inv, v[4 * q4 + 2] * inv, v[4 * q4 + 3] * inv);
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

  // ---- teardown: TMEM back, then a bounded handshake so that neither CTA of the
  // pair exits while the other may still write into its shared memory
  if (warp < 4 && lane == 0) bulk_wait_read_all();   // my last sends have left my shared memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  if (tid == 0) {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
    remote_arrive(map_remote(smem_u32(&bar[kDone]), peer));
    volatile int never = 0;
    mbar_wait_cluster(&bar[kDone], 0, &never);
  }
  __syncthreads();
}

}  // namespace pa
