// pa_api.cu -- C ABI of libpa_b200: argument validation, work planning, TMA
// descriptor set-up and kernel launches.  See include/pa.h for the contract.
//
// Everything here runs on the host and is asynchronous with respect to the GPU:
// no call synchronises, copies device data to the host or allocates memory
// (pa_device_status is the one documented exception: it synchronises).
#include "pa.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <atomic>
#include <mutex>

#include "pa_gqa.cuh"
#include "pa_merge.cuh"
#include "pa_mla.cuh"

namespace {

constexpr int kMaxBatch = 4096;            // prefix table lives in shared memory
constexpr int kMaxBatchMla = 32768;        // the merge's prefix table: 128 KB of shared memory
// Empty units at the start of every non-empty segment of a GQA stream: the
// per-segment cost (query switch, partial or output rows, the first tile's
// wait) in tiles, so that equal pieces take equal time on mixed lengths.
constexpr int kSegUnits = 2;
constexpr int kMaxPartitions = 1 << 20;
constexpr float kLog2e = 1.4426950408889634f;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ driver entry

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Row-major [rows][inner] 16-bit tensor, boxes of box_rows x box_inner, 128 B swizzle.
bool make_map_2d(CUtensorMap *m, const void *base, bool bf16, uint64_t inner, uint64_t rows,
                 uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows][128] 16-bit tensor viewed as (64 elements, rows, 2 halves),
// the halves 128 bytes apart: one box of 64 x box_rows x 2 lands as
// [2][box_rows][64] with 128 B swizzle, the layout two 64-wide 2-D boxes give.
bool make_map_3d_halves(CUtensorMap *m, const void *base, bool bf16, uint64_t rows,
                        uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MLA latent pool (or query) [rows][576] bf16 viewed as (64 dims, rows, 9 slabs): the slabs
// are 128 bytes apart in a row.  A box of 64 x box_rows x box_slabs lands as
// [box_slabs][box_rows][64] with 128 B swizzle: whole slabs of a token range, in
// the layout that 2-D boxes of one 64-dim slab give one slab at a time.
bool make_map_latent_slabs(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows,
                           uint32_t box_slabs) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, pa::kMlaDk / 64};
  cuuint64_t strides[2] = {pa::kMlaDk * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_slabs};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Float8 KV cache: one byte per element, rows of `inner` bytes.
bool make_map_2d_u8(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows,
                    uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

// Resident CTAs per SM of `kernel` with `smem` dynamic bytes, after raising the
// kernel's dynamic shared-memory limit (once per device is enough; it is cheap).
int resident_ctas(const void *kernel, int threads, size_t smem) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return -1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
    return -1;
  return n;
}

// ------------------------------------------------------------------ GQA variants

// Kernel modes: 16-bit cache, float8 cache, index-list decode, 16-bit cache with
// the single-pass merge.
enum GqaMode { kMode16 = 0, kModeKv8 = 1, kModeIndexed = 2, kModeFused = 3 };

template <int D, int NT, bool BF16, int MODE>
struct GqaVariant {
  // 192 KB of rings per CTA: 8 warps x 3 x 8 KB (D 128), 8 x 6 x 4 KB (D 64, or
  // float8 at 16 heads per group), 12 x 4 x 4 KB (float8 up to 8 heads per group),
  // 12 x 2 x 8 KB (index list up to 8 heads per group)
  static constexpr int W = pa::gqa_warps(MODE, NT);
  static constexpr int R = MODE == kModeKv8       ? (W == 12 ? 4 : 6)
                           : MODE == kModeIndexed ? (W == 12 ? 2 : 3)
                                                  : (D == 128 ? 3 : 6);
  using L = pa::GqaLayout<D, NT, R, MODE, W>;
  static const void *kernel() {
    return reinterpret_cast<const void *>(&pa::gqa_decode_kernel<D, NT, BF16, R, MODE, W>);
  }
  static void launch(int grid, size_t smem, cudaStream_t st, const CUtensorMap &k,
                     const CUtensorMap &v, const pa::GqaParams &p) {
    pa::gqa_decode_kernel<D, NT, BF16, R, MODE, W><<<grid, 32 * W, smem, st>>>(k, v, p);
  }
};

template <template <int, int, bool, int> class F, typename... A>
bool dispatch_gqa(int D, int NT, bool bf16, int mode, A &&...a) {
#define PA_CASE(d, nt, b, m)                                \
  if (D == d && NT == nt && bf16 == b && mode == m) {       \
    F<d, nt, b, m>::run(static_cast<A &&>(a)...);           \
    return true;                                            \
  }
  PA_CASE(128, 1, true, 0) PA_CASE(128, 1, false, 0) PA_CASE(128, 2, true, 0)
  PA_CASE(128, 2, false, 0) PA_CASE(64, 1, true, 0) PA_CASE(64, 1, false, 0)
  PA_CASE(64, 2, true, 0) PA_CASE(64, 2, false, 0)
  PA_CASE(128, 1, true, 1) PA_CASE(128, 1, false, 1) PA_CASE(128, 2, true, 1)
  PA_CASE(128, 2, false, 1)
  PA_CASE(128, 1, true, 2) PA_CASE(128, 1, false, 2) PA_CASE(128, 2, true, 2)
  PA_CASE(128, 2, false, 2)
  PA_CASE(128, 1, true, 3) PA_CASE(128, 1, false, 3) PA_CASE(128, 2, true, 3)
  PA_CASE(128, 2, false, 3) PA_CASE(64, 1, true, 3) PA_CASE(64, 1, false, 3)
  PA_CASE(64, 2, true, 3) PA_CASE(64, 2, false, 3)
#undef PA_CASE
  return false;
}

template <int D, int NT, bool BF16, int MODE>
struct QueryResident {
  static void run(int B, int *out) {
    using V = GqaVariant<D, NT, BF16, MODE>;
    *out = resident_ctas(V::kernel(), 32 * V::W, V::L::bytes(B));
  }
};

struct GqaPlan {
  int G = 0, NT = 0, parts = 0, warps = pa::kWarps;
  size_t off_lse = 0, off_o = 0, off_ctr = 0, bytes = 0;
};

int default_gqa_parts(int D, int NT, bool bf16, int mode, int B) {
  const int sms = sm_count();
  if (sms <= 0) return -1;
  int per = -1;
  if (!dispatch_gqa<QueryResident>(D, NT, bf16, mode, B, &per) || per <= 0) return -1;
  return sms * per;
}

pa_status plan_gqa(const pa_desc *d, GqaPlan *pl, int mode = kMode16) {
  if (!d) return PA_ERR_INVALID_ARG;
  if (d->batch < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0 ||
      d->block_size <= 0 || d->max_blocks_per_seq <= 0 || d->num_blocks <= 0 ||
      d->num_partitions < 0 || d->num_partitions > kMaxPartitions)
    return PA_ERR_INVALID_ARG;
  if (d->dtype != PA_F16 && d->dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = d->num_q_heads / d->num_kv_heads;
  if (G > 16) return PA_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if ((mode == kModeKv8 || mode == kModeIndexed) && d->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (d->block_size % pa::kTile || d->block_size > 1024) return PA_ERR_UNSUPPORTED;
  if (d->batch > kMaxBatch) return PA_ERR_UNSUPPORTED;
  const int64_t kv_rows = int64_t(d->num_blocks) * d->num_kv_heads * d->block_size;
  const int64_t q_rows = int64_t(d->batch) * d->num_q_heads;
  const int64_t cap = int64_t(d->max_blocks_per_seq) * d->block_size;
  // work units of the flattened stream: tiles plus kSegUnits per segment
  const int64_t max_tiles = int64_t(d->batch) * (cap / pa::kTile + kSegUnits) * d->num_kv_heads;
  if (kv_rows > INT32_MAX || q_rows > INT32_MAX || cap > INT32_MAX || max_tiles > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  pl->G = G;
  pl->NT = G <= 8 ? 1 : 2;
  pl->parts = d->num_partitions;
  if (pl->parts == 0) {
    pl->parts = default_gqa_parts(d->head_dim, pl->NT, d->dtype == PA_BF16, mode, d->batch);
    if (pl->parts <= 0) return PA_ERR_CUDA;
  }
  // one partial slot per (warp piece, segment) pair a piece can end: piece + segment
  pl->warps = pa::gqa_warps(mode, pl->NT);
  const size_t slots = size_t(pl->parts) * pl->warps + size_t(d->batch) * d->num_kv_heads;
  pl->off_lse = 0;
  pl->off_o = pl->off_lse + round_up(slots * G * 4, 256);
  // arrival counters of the single-pass merge, one 64-bit word per segment
  pl->off_ctr = round_up(pl->off_o + slots * G * size_t(d->head_dim) * 4, 256);
  pl->bytes = pl->off_ctr + size_t(d->batch) * d->num_kv_heads * 8;
  return PA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status check_gqa_args(const pa_desc *d, const GqaPlan &pl, const void *q, const void *k,
                         const void *v, const int32_t *bt, const int32_t *cl, const void *out,
                         const void *ws, size_t ws_bytes) {
  if (!q || !k || !v || !bt || !cl || !out) return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(bt) & 3u) || (reinterpret_cast<uintptr_t>(cl) & 3u))
    return PA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < pl.bytes) return PA_ERR_WORKSPACE;
  (void)d;
  return PA_OK;
}

template <int D, int NT, bool BF16, int MODE>
struct LaunchPartition {
  static void run(int grid, cudaStream_t st, const CUtensorMap *maps, const pa::GqaParams *p,
                  cudaError_t *err) {
    using V = GqaVariant<D, NT, BF16, MODE>;
    const size_t smem = V::L::bytes(p->B);
    *err = cudaFuncSetAttribute(V::kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem));
    if (*err != cudaSuccess) return;
    V::launch(grid, smem, st, maps[0], maps[1], *p);
    *err = cudaGetLastError();
  }
};

// The merge kernel for value width DV, launched with programmatic dependent
// launch so that its CTAs can be scheduled while the partition grid drains.
// A merge CTA holds the tile prefix [B + 1] in dynamic shared memory; past the
// 48 KB default the kernel's limit is raised first.
cudaError_t merge_smem_limit(const void *kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <int DV, bool BF16>
cudaError_t launch_merge(const pa::MergeParams &mp, int segments, cudaStream_t st) {
  const cudaError_t e = merge_smem_limit(reinterpret_cast<const void *>(&pa::merge_kernel<DV, BF16>),
                                         pa::merge_smem_bytes(mp.B));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(segments), static_cast<unsigned>(mp.G), 1);
  cfg.blockDim = dim3(pa::kMergeThreads, 1, 1);
  cfg.dynamicSmemBytes = pa::merge_smem_bytes(mp.B);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::merge_kernel<DV, BF16>, mp);
}

// Warp-per-row merge: one warp per (segment, head) row, 8 rows per CTA.
template <int DV, bool BF16>
cudaError_t launch_merge_rows(const pa::MergeParams &mp, int segments, cudaStream_t st) {
  const cudaError_t e = merge_smem_limit(
      reinterpret_cast<const void *>(&pa::merge_rows_kernel<DV, BF16>), pa::merge_smem_bytes(mp.B));
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(segments) * mp.G;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + pa::kMergeRowsPerCta - 1) / pa::kMergeRowsPerCta),
                     1, 1);
  cfg.blockDim = dim3(pa::kMergeRowsPerCta * 32, 1, 1);
  cfg.dynamicSmemBytes = pa::merge_smem_bytes(mp.B);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pa::merge_rows_kernel<DV, BF16>, mp);
}

// Few pieces per segment (short and mixed contexts, MLA): a warp per row keeps
// every row's loads to two round trips.  Many pieces per segment (one long
// context spread over the GPU): a CTA per row, whose eight piece groups load in
// parallel, is faster.
constexpr int kRowsMergeMaxPieces = 8;

cudaError_t merge_dispatch(int DV, bool bf16, const pa::MergeParams &mp, int segments,
                           cudaStream_t st) {
  if (static_cast<long long>(mp.pieces) <= static_cast<long long>(kRowsMergeMaxPieces) * segments) {
    if (DV == 128) return bf16 ? launch_merge_rows<128, true>(mp, segments, st)
                               : launch_merge_rows<128, false>(mp, segments, st);
    if (DV == 512) return bf16 ? launch_merge_rows<512, true>(mp, segments, st)
                               : launch_merge_rows<512, false>(mp, segments, st);
  }
  if (DV == 128) return bf16 ? launch_merge<128, true>(mp, segments, st)
                             : launch_merge<128, false>(mp, segments, st);
  if (DV == 64) return bf16 ? launch_merge<64, true>(mp, segments, st)
                            : launch_merge<64, false>(mp, segments, st);
  if (DV == 512) return bf16 ? launch_merge<512, true>(mp, segments, st)
                             : launch_merge<512, false>(mp, segments, st);
  return cudaErrorInvalidValue;
}

// An automatic launch (num_partitions == 0) sizes its grid for a full GPU but
// does not cut a short tile stream into pieces much smaller than the partial
// output each piece writes: a piece leaves G x D fp32 (GQA: one 16-token K+V tile
// is 16 x D x 4 bytes, so G tiles per piece keep partials at or below the KV
// bytes read; at least 2) or 128 x 512 fp32 (MLA: 11 work units of 96-token tiles).  A
// single short sequence or a single kv head would otherwise spend more on
// partials and their merge than on the KV.  An explicit partition count is used
// as given.
int min_tiles_gqa(int G) { return G > 2 ? G : 2; }
constexpr int kMinTilesMla = 11;  // tiles of 96 tokens

// kFused: the partition kernel also merges (the last piece of each split segment),
// so no merge grid is launched
enum Pass { kPartition = 1, kMerge = 2, kBoth = 3, kFused = 4 };

// Epoch of a single-pass call: tags the workspace's arrival counters so that words
// left by another call (or never written) count as zero; never 0 (0 = not fused).
uint32_t next_epoch() {
  static std::atomic<uint32_t> epoch{0};
  uint32_t e;
  do e = epoch.fetch_add(1, std::memory_order_relaxed) + 1; while (e == 0);
  return e;
}

// mode kModeKv8: k / v hold float8 E4M3 codes, key = code x k_scale, value =
// code x v_scale.  kModeIndexed: cl holds the selected counts and token_index
// [B][max_sel] the selected positions.
pa_status run_gqa(int passes, const pa_desc *d, const void *q, const void *k, const void *v,
                  const int32_t *bt, const int32_t *cl, float scale, void *out, void *ws,
                  size_t ws_bytes, void *stream, int mode = kMode16, float k_scale = 1.f,
                  float v_scale = 1.f, const int32_t *token_index = nullptr, int max_sel = 0) {
  if (passes & kFused) mode = kModeFused;
  const bool kv8 = mode == kModeKv8;
  GqaPlan pl;
  pa_status s = plan_gqa(d, &pl, mode);
  if (s != PA_OK) return s;
  if (d->batch == 0) return PA_OK;
  s = check_gqa_args(d, pl, q, k, v, bt, cl, out, ws, ws_bytes);
  if (s != PA_OK) return s;
  if (!std::isfinite(scale) || !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return PA_ERR_INVALID_ARG;
  if (mode == kModeIndexed &&
      (!token_index || (reinterpret_cast<uintptr_t>(token_index) & 3u) || max_sel <= 0))
    return PA_ERR_INVALID_ARG;
  // the index-list stream counts tiles of up to max_sel entries per sequence
  if (mode == kModeIndexed &&
      int64_t(d->batch) * (max_sel / pa::kTile + 1) * d->num_kv_heads > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(ws);
  const bool bf16 = d->dtype == PA_BF16;
  const int D = d->head_dim;

  if (passes & kPartition) {
    CUtensorMap maps[2];
    const uint64_t kv_rows = uint64_t(d->num_blocks) * d->num_kv_heads * d->block_size;
    const bool mapped =
        kv8 ? make_map_2d_u8(&maps[0], k, D, kv_rows, D, pa::kTile) &&
                  make_map_2d_u8(&maps[1], v, D, kv_rows, D, pa::kTile)
        : D == 128 ? make_map_3d_halves(&maps[0], k, bf16, kv_rows, pa::kTile) &&
                         make_map_3d_halves(&maps[1], v, bf16, kv_rows, pa::kTile)
            : make_map_2d(&maps[0], k, bf16, D, kv_rows, 64, pa::kTile) &&
                  make_map_2d(&maps[1], v, bf16, D, kv_rows, 64, pa::kTile);
    if (!mapped) return PA_ERR_CUDA;
    pa::GqaParams p;
    p.q = static_cast<const uint16_t *>(q);
    p.block_table = bt;
    p.context_lens = cl;
    p.out = out;
    p.part_o = reinterpret_cast<float *>(w + pl.off_o);
    p.part_lse = reinterpret_cast<float *>(w + pl.off_lse);
    p.B = d->batch;
    p.Hq = d->num_q_heads;
    p.Hkv = d->num_kv_heads;
    p.G = pl.G;
    p.bs = d->block_size;
    p.mbs = d->max_blocks_per_seq;
    p.nb = d->num_blocks;
    p.tiles_per_block = d->block_size / pa::kTile;
    p.parts = pl.parts;
    p.scale_log2 = scale * k_scale * kLog2e;
    p.v_scale = v_scale;
    p.token_index = token_index;
    p.max_sel = max_sel;
    p.k_cache = k;
    p.v_cache = v;
    p.min_tiles = d->num_partitions == 0 ? min_tiles_gqa(pl.G) : 0;
    p.seg_ctr = reinterpret_cast<unsigned long long *>(w + pl.off_ctr);
    p.seg_units = mode == kModeIndexed ? 0 : kSegUnits;
    p.epoch = mode == kModeFused ? next_epoch() : 0u;
    cudaError_t err = cudaSuccess;
    if (!dispatch_gqa<LaunchPartition>(D, pl.NT, bf16, mode, pl.parts, st, maps, &p, &err))
      return PA_ERR_UNSUPPORTED;
    if (err != cudaSuccess) return PA_ERR_CUDA;
  }
  if (passes & kMerge) {
    pa::MergeParams mp;
    mp.part_o = reinterpret_cast<const float *>(w + pl.off_o);
    mp.part_lse = reinterpret_cast<const float *>(w + pl.off_lse);
    mp.lens = cl;
    mp.cap = mode == kModeIndexed ? max_sel : d->max_blocks_per_seq * d->block_size;
    mp.tile = pa::kTile;
    mp.seg_units = mode == kModeIndexed ? 0 : kSegUnits;
    mp.out = out;
    mp.B = d->batch;
    mp.Hq = d->num_q_heads;
    mp.Hkv = d->num_kv_heads;
    mp.G = pl.G;
    mp.pieces = pl.parts * pl.warps;
    mp.min_tiles = d->num_partitions == 0 ? min_tiles_gqa(pl.G) : 0;
    mp.floor_pieces = static_cast<long long>(pl.warps) * d->batch * d->num_kv_heads;
    if (merge_dispatch(D, bf16, mp, d->batch * d->num_kv_heads, st) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

// ------------------------------------------------------------------ MLA

struct MlaPlan {
  int parts = 0;
  size_t off_lse = 0, off_o = 0, bytes = 0;
};

// Launch configuration of the MLA partition pass: clusters of two CTAs (one CTA
// pair per piece), one CTA per SM by its shared memory.
cudaLaunchConfig_t mla_launch_config(int parts, cudaStream_t st, cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * parts), 1, 1);
  cfg.blockDim = dim3(pa::kMlaThreads, 1, 1);
  cfg.dynamicSmemBytes = pa::MlaLayout::bytes();
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Pieces (CTA pairs) that can all be resident at once: a pair must fit on two
// SMs of one GPU processing cluster, so this can be fewer than SMs / 2.
int default_mla_parts() {
  const size_t smem = pa::MlaLayout::bytes();
  if (cudaFuncSetAttribute(pa::mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return -1;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = mla_launch_config(1, nullptr, attr);
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, pa::mla_decode_kernel, &cfg) != cudaSuccess ||
      clusters <= 0) {
    const int sms = sm_count();
    return sms >= 2 ? sms / 2 : -1;
  }
  return clusters;
}

pa_status plan_mla(const pa_mla_desc *d, MlaPlan *pl) {
  if (!d) return PA_ERR_INVALID_ARG;
  if (d->batch < 0 || d->num_heads <= 0 || d->kv_dim <= 0 || d->v_dim <= 0 ||
      d->block_size <= 0 || d->max_blocks_per_seq <= 0 || d->num_blocks <= 0 ||
      d->num_partitions < 0 || d->num_partitions > kMaxPartitions)
    return PA_ERR_INVALID_ARG;
  if (d->dtype != PA_F16 && d->dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (d->v_dim > d->kv_dim) return PA_ERR_INVALID_ARG;
  if (d->num_heads != pa::kMlaHeads || d->kv_dim != pa::kMlaDk || d->v_dim != pa::kMlaDv ||
      d->dtype != PA_BF16)
    return PA_ERR_UNSUPPORTED;
  if (d->block_size % pa::kMlaBox || d->block_size > 1024) return PA_ERR_UNSUPPORTED;
  if (d->batch > kMaxBatchMla) return PA_ERR_UNSUPPORTED;
  const int64_t rows = int64_t(d->num_blocks) * d->block_size;
  const int64_t cap = int64_t(d->max_blocks_per_seq) * d->block_size;
  if (rows > INT32_MAX || cap > INT32_MAX || int64_t(d->batch) * pa::kMlaHeads > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  pl->parts = d->num_partitions;
  if (pl->parts == 0) {
    pl->parts = default_mla_parts();
    if (pl->parts <= 0) return PA_ERR_CUDA;
  }
  const size_t slots = size_t(pl->parts) + size_t(d->batch);
  pl->off_lse = 0;
  pl->off_o = pl->off_lse + round_up(slots * pa::kMlaHeads * 4, 256);
  pl->bytes = pl->off_o + slots * pa::kMlaHeads * size_t(pa::kMlaDv) * 4;
  return PA_OK;
}

pa_status run_mla(int passes, const pa_mla_desc *d, const void *q, const void *lat,
                  const int32_t *bt, const int32_t *cl, float scale, void *out, void *ws,
                  size_t ws_bytes, void *stream) {
  MlaPlan pl;
  pa_status s = plan_mla(d, &pl);
  if (s != PA_OK) return s;
  if (d->batch == 0) return PA_OK;
  if (!q || !lat || !bt || !cl || !out) return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(lat) || !aligned16(out)) return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(bt) & 3u) || (reinterpret_cast<uintptr_t>(cl) & 3u))
    return PA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < pl.bytes) return PA_ERR_WORKSPACE;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(ws);

  if (passes & kPartition) {
    // A CTA's 48 tokens of a tile: one 3-D box of whole slabs when they lie in one
    // block, else 2-D boxes of 16 or 32 rows of one 64-dim slab each (block sizes
    // are multiples of 16, so no 16-row group crosses a block)
    CUtensorMap ta, ta32, tw9, tw2;
    const uint64_t rows = uint64_t(d->num_blocks) * d->block_size;
    if (!make_map_2d(&ta, lat, true, pa::kMlaDk, rows, 64, pa::kMlaBox) ||
        !make_map_2d(&ta32, lat, true, pa::kMlaDk, rows, 64, 2 * pa::kMlaBox) ||
        !make_map_latent_slabs(&tw9, lat, rows, pa::kMlaHalf, pa::MlaLayout::kSlabs) ||
        !make_map_latent_slabs(&tw2, lat, rows, pa::kMlaHalf, 2))
      return PA_ERR_CUDA;
    // the query [B * 128 heads][576] in the same slab view: a 64-head x 4-slab box
    // is the shared-memory part of the score MMA's A operand
    CUtensorMap tq;
    if (!make_map_latent_slabs(&tq, q, uint64_t(d->batch) * pa::kMlaHeads, 64,
                               pa::MlaLayout::kQSlabs))
      return PA_ERR_CUDA;
    pa::MlaParams p;
    p.q = static_cast<const uint16_t *>(q);
    p.lat = static_cast<const uint16_t *>(lat);
    p.block_table = bt;
    p.context_lens = cl;
    p.out = out;
    p.part_o = reinterpret_cast<float *>(w + pl.off_o);
    p.part_lse = reinterpret_cast<float *>(w + pl.off_lse);
    p.B = d->batch;
    p.bs = d->block_size;
    p.mbs = d->max_blocks_per_seq;
    p.nb = d->num_blocks;
    p.parts = pl.parts;
    p.min_tiles = d->num_partitions == 0 ? kMinTilesMla : 0;
    p.scale_log2 = scale * kLog2e;
    const size_t smem = pa::MlaLayout::bytes();
    if (cudaFuncSetAttribute(pa::mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return PA_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = mla_launch_config(pl.parts, st, attr);
    if (cudaLaunchKernelEx(&cfg, pa::mla_decode_kernel, ta, ta32, tw9, tw2, tq, p) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (passes & kMerge) {
    pa::MergeParams mp;
    mp.part_o = reinterpret_cast<const float *>(w + pl.off_o);
    mp.part_lse = reinterpret_cast<const float *>(w + pl.off_lse);
    mp.lens = cl;
    mp.cap = d->max_blocks_per_seq * d->block_size;
    mp.tile = pa::kMlaTile;
    mp.seg_units = pa::kMlaSeqUnits;
    mp.out = out;
    mp.B = d->batch;
    mp.Hq = pa::kMlaHeads;
    mp.Hkv = 1;
    mp.G = pa::kMlaHeads;
    mp.pieces = pl.parts;
    mp.min_tiles = d->num_partitions == 0 ? kMinTilesMla : 0;
    mp.floor_pieces = d->batch;
    if (merge_dispatch(pa::kMlaDv, true, mp, d->batch, st) != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace

// ==================================================================== C ABI

extern "C" {

size_t pa_workspace_size(const pa_desc *desc) {
  GqaPlan pl;
  if (plan_gqa(desc, &pl) != PA_OK) return 0;
  size_t bytes = pl.bytes;
  // the float8 and index-list calls may launch another grid size
  for (int mode : {kModeKv8, kModeIndexed, kModeFused}) {
    GqaPlan other;
    if ((mode == kModeFused || desc->head_dim == 128) && plan_gqa(desc, &other, mode) == PA_OK &&
        other.bytes > bytes)
      bytes = other.bytes;
  }
  return bytes;
}

pa_status pa_decode_kv_e4m3(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *context_lens, float scale, float k_scale,
                            float v_scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kBoth, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream, kModeKv8, k_scale, v_scale);
}

pa_status pa_decode_kv_e4m3_partition(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *context_lens, float scale, float k_scale,
                            float v_scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kPartition, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream, kModeKv8, k_scale, v_scale);
}

pa_status pa_decode_kv_e4m3_merge(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *context_lens, float scale, float k_scale,
                            float v_scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kMerge, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream, kModeKv8, k_scale, v_scale);
}

pa_status pa_decode_indexed(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *token_index, int max_sel, const int32_t *n_sel,
                            float scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kBoth, desc, q, k_cache, v_cache, block_table, n_sel, scale, out, workspace,
                 workspace_bytes, stream, kModeIndexed, 1.f, 1.f, token_index, max_sel);
}

pa_status pa_decode_indexed_partition(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *token_index, int max_sel, const int32_t *n_sel,
                            float scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kPartition, desc, q, k_cache, v_cache, block_table, n_sel, scale, out, workspace,
                 workspace_bytes, stream, kModeIndexed, 1.f, 1.f, token_index, max_sel);
}

pa_status pa_decode_indexed_merge(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *token_index, int max_sel, const int32_t *n_sel,
                            float scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream) {
  return run_gqa(kMerge, desc, q, k_cache, v_cache, block_table, n_sel, scale, out, workspace,
                 workspace_bytes, stream, kModeIndexed, 1.f, 1.f, token_index, max_sel);
}

pa_status pa_decode(const pa_desc *desc, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_table, const int32_t *context_lens, float scale,
                    void *out, void *workspace, size_t workspace_bytes, void *stream) {
  return run_gqa(kBoth, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream);
}

pa_status pa_decode_fused(const pa_desc *desc, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *block_table,
                          const int32_t *context_lens, float scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream) {
  return run_gqa(kPartition | kFused, desc, q, k_cache, v_cache, block_table, context_lens, scale,
                 out, workspace, workspace_bytes, stream);
}

pa_status pa_decode_partition(const pa_desc *desc, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *block_table,
                              const int32_t *context_lens, float scale, void *out,
                              void *workspace, size_t workspace_bytes, void *stream) {
  return run_gqa(kPartition, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream);
}

pa_status pa_decode_merge(const pa_desc *desc, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *block_table,
                          const int32_t *context_lens, float scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream) {
  return run_gqa(kMerge, desc, q, k_cache, v_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream);
}

size_t pa_mla_workspace_size(const pa_mla_desc *desc) {
  MlaPlan pl;
  if (plan_mla(desc, &pl) != PA_OK) return 0;
  return pl.bytes;
}

pa_status pa_decode_mla(const pa_mla_desc *desc, const void *q, const void *latent_cache,
                        const int32_t *block_table, const int32_t *context_lens, float scale,
                        void *out, void *workspace, size_t workspace_bytes, void *stream) {
  return run_mla(kBoth, desc, q, latent_cache, block_table, context_lens, scale, out, workspace,
                 workspace_bytes, stream);
}

pa_status pa_decode_mla_partition(const pa_mla_desc *desc, const void *q,
                                  const void *latent_cache, const int32_t *block_table,
                                  const int32_t *context_lens, float scale, void *out,
                                  void *workspace, size_t workspace_bytes, void *stream) {
  return run_mla(kPartition, desc, q, latent_cache, block_table, context_lens, scale, out,
                 workspace, workspace_bytes, stream);
}

pa_status pa_decode_mla_merge(const pa_mla_desc *desc, const void *q, const void *latent_cache,
                              const int32_t *block_table, const int32_t *context_lens,
                              float scale, void *out, void *workspace, size_t workspace_bytes,
                              void *stream) {
  return run_mla(kMerge, desc, q, latent_cache, block_table, context_lens, scale, out, workspace,
                 workspace_bytes, stream);
}

int pa_default_partitions(int kind, int head_dim) {
  if (kind == 0) {
    if (head_dim != 64 && head_dim != 128) return -1;
    return default_gqa_parts(head_dim, 1, true, kMode16, 256);
  }
  if (kind == 2) return head_dim == 128 ? default_gqa_parts(128, 1, true, kModeKv8, 256) : -1;
  if (kind == 3) return head_dim == 128 ? default_gqa_parts(128, 1, true, kModeIndexed, 256) : -1;
  return default_mla_parts();
}

void pa_test_inject_stall(int enable) {
  const int v = enable ? 1 : 0;
  (void)cudaMemcpyToSymbol(pa::g_stall_test, &v, sizeof(int));
}

pa_status pa_device_status(void *stream, int reset) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_status, sizeof(int)) != cudaSuccess) return PA_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_status, &zero, sizeof(int)) != cudaSuccess) return PA_ERR_CUDA;
  }
  return static_cast<pa_status>(v);
}

const char *pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_BAD_BLOCK_ID: return "block id or context length outside the data contract";
    case PA_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_TOO_LARGE: return "call needs more scratch than the static buffer holds";
  }
  return "unknown status";
}

}  // extern "C"

// ==================================================================== allocation-free entry

// Scratch of pa_decode_static: a fixed device buffer in the library itself, for
// callers that cannot allocate device memory.  Host code must not pass the
// symbol itself to a kernel (on the host it names a shadow variable, not device
// memory); its device address is looked up below, once per CUDA context (one per
// device unless the device is reset).
static __device__ __align__(256) unsigned char g_pa_static_scratch[PA_STATIC_SCRATCH_BYTES];

namespace {

// The address is valid in the CUDA context it was looked up in.  A device reset
// destroys that context (and a driver-API caller may make another one current),
// so the cache is keyed by the unique id of the current context (cuCtxGetId),
// never by the device ordinal: a context created after a reset gets a new id and
// a fresh lookup.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name) {
  void *ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &ptr, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(ptr);
}

// Unique id of the calling thread's current context, or 0 if there is none.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

constexpr int kMaxContexts = 64;
std::mutex g_static_mu;
unsigned long long g_static_ctx[kMaxContexts] = {};
void *g_static_ptr[kMaxContexts] = {};
int g_static_n = 0;

// Device address of the static scratch in the current context (looked up on the
// first call in each context), or nullptr on error.
void *static_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_mu);
  unsigned long long id = current_context_id();
  for (int i = 0; id != 0 && i < g_static_n; ++i)
    if (g_static_ctx[i] == id) return g_static_ptr[i];
  // with no context current yet, the lookup makes the device's primary one current
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_pa_static_scratch) != cudaSuccess || !ptr) return nullptr;
  if (id == 0) id = current_context_id();
  if (id != 0 && g_static_n < kMaxContexts) {
    g_static_ctx[g_static_n] = id;
    g_static_ptr[g_static_n] = ptr;
    ++g_static_n;
  }
  return ptr;
}

}  // namespace

extern "C" pa_status pa_decode_static(const pa_desc *desc, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_table,
                                      const int32_t *context_lens, float scale, void *out,
                                      void *stream) {
  GqaPlan pl;
  pa_status s = plan_gqa(desc, &pl);
  if (s != PA_OK) return s;
  if (desc->batch == 0) return PA_OK;
  if (pl.bytes > PA_STATIC_SCRATCH_BYTES) return PA_ERR_TOO_LARGE;
  void *scratch = static_scratch_address();
  if (!scratch) return PA_ERR_CUDA;
  return run_gqa(kBoth, desc, q, k_cache, v_cache, block_table, context_lens, scale, out, scratch,
                 PA_STATIC_SCRATCH_BYTES, stream);
}
