/*
 * pa.h -- C ABI of the B200 paged split-KV decode attention library (libpa_b200.so).
 *
 * One operation: single-query-token decode attention over a block-paged KV
 * cache, computed Flash-Decoding style.
 *
 *   out[b, h, :] = softmax_t( scale * q[b, h, :] . K_b[t, :] ) V_b[t, :],  t < context_lens[b]
 *
 * where logical token t of sequence b lives in row t % block_size of physical
 * block block_table[b][t / block_size] (page "wenku.it search: paged attention",
 * vLLM PagedAttention snippet on paged key/value memory).  The KV stream of every
 * (sequence, kv head) is split along the sequence; each piece is attended
 * separately, recording the log-sum-exp of each softmax row, and the pieces are
 * rescaled and reduced at the end (page "cidian.kuaisou.com: flash decoding ++",
 * snippets on the three Flash-Decoding steps and on loading K/V in parallel then
 * rescaling and combining).  Query head h reads kv head h / (Hq / Hkv) (grouped
 * query heads share one kv head, page "bjpcjp.github.io: llms-attention",
 * MHA -> GQA -> MLA teaser).  The MLA entry points read one shared latent row per
 * token: the key is the whole kv_dim-wide row and the value its first v_dim dims
 * (page "wenku.it search: Multi-head Latent Attention (MLA)", DeepSeek-V2
 * abstract on the compressed latent KV).
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or retains them.  All are dense row-major:
 *       q            [batch][num_q_heads][head_dim]                 dtype
 *       k_cache      [num_blocks][num_kv_heads][block_size][head_dim]  dtype
 *       v_cache      [num_blocks][num_kv_heads][block_size][head_dim]  dtype
 *       block_table  [batch][max_blocks_per_seq]                    int32
 *       context_lens [batch]                                        int32
 *       out          [batch][num_q_heads][head_dim]                 dtype
 *     MLA: q [batch][num_heads][kv_dim], latent_cache [num_blocks][block_size][kv_dim],
 *          out [batch][num_heads][v_dim].
 *     Base addresses must be 16-byte aligned.
 *   - workspace is caller-owned device scratch of at least the size returned by
 *     the matching *_workspace_size call; its contents need no initialisation
 *     and are overwritten by every call.  Two calls in flight at the same time
 *     must not share a workspace.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on it; nothing is synchronised and no host-side
 *     copy of device data is made.  context_lens and block_table are read only by
 *     the GPU.
 *   - Data contract (checked on the GPU; a violation skips the offending load and
 *     records an error readable through pa_device_status):
 *       0 <= context_lens[b] <= max_blocks_per_seq * block_size,
 *       0 <= block_table[b][j] < num_blocks for j < ceil(context_lens[b] / block_size).
 *     Entries past ceil(context_lens[b] / block_size) are never read.
 *     context_lens[b] == 0 gives an all-zero output row.
 *   - Errors are returned, never thrown; nothing is printed.  Argument errors are
 *     detected before any launch.  The library keeps no per-call state; it is
 *     safe to call from several host threads on different streams.
 */
#ifndef PA_B200_H
#define PA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
  PA_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim, block_size, group size */
  PA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, no device) */
  PA_ERR_BAD_BLOCK_ID = 4,  /* device: block id or context length outside the contract */
  PA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out */
  PA_ERR_WORKSPACE = 6,     /* workspace null or smaller than required */
  PA_ERR_TOO_LARGE = 7      /* pa_decode_static: the call needs more scratch than the
                               library's fixed device buffer holds */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Shape of a GQA / MHA / MQA decode call.
 * Supported: head_dim in {64, 128}; block_size a multiple of 16 up to 1024;
 * 1 <= num_q_heads / num_kv_heads <= 16; 0 <= batch <= 4096 (0 is a no-op).
 * num_partitions: CTAs of the partition grid; the flattened KV stream is cut into
 * equal-work pieces, one per warp: 8 per CTA (12 in pa_decode_kv_e4m3 and
 * pa_decode_indexed at up to 8 query heads per kv head).  0 picks (SM count) x (resident CTAs
 * per SM) for the current device, with pieces no shorter than the partial output
 * they write. */
typedef struct {
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;
  pa_dtype dtype;
  int num_partitions;
} pa_desc;

/* Shape of an MLA absorbed decode call.  Supported: num_heads 128, kv_dim 576,
 * v_dim 512, block_size a multiple of 16 up to 1024, dtype PA_BF16,
 * 0 <= batch <= 32768.
 * num_partitions counts CTA pairs (0 = as many as can be resident). */
typedef struct {
  int batch;
  int num_heads;
  int kv_dim;
  int v_dim;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;
  pa_dtype dtype;
  int num_partitions;
} pa_mla_desc;

/* Workspace bytes a pa_decode call with this descriptor needs; 0 if the
 * descriptor is invalid or (num_partitions == 0 and no CUDA device is usable). */
size_t pa_workspace_size(const pa_desc *desc);

/* Full decode step on `stream`: the partition kernel, then the LSE merge kernel
 * (launched with programmatic dependent launch so that it overlaps the
 * partition kernel's tail). */
pa_status pa_decode(const pa_desc *desc, const void *q, const void *k_cache,
                    const void *v_cache, const int32_t *block_table,
                    const int32_t *context_lens, float scale, void *out, void *workspace,
                    size_t workspace_bytes, void *stream);

/* The two kernels of pa_decode, exposed separately so that each can be timed on
 * its own: pa_decode_partition runs the partition pass (writes the output of
 * every (sequence, kv head) that one piece covered, and partials for the rest);
 * pa_decode_merge combines the partials.  pa_decode_merge must follow
 * pa_decode_partition on the same stream with the same arguments and workspace. */
pa_status pa_decode_partition(const pa_desc *desc, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *block_table,
                              const int32_t *context_lens, float scale, void *out,
                              void *workspace, size_t workspace_bytes, void *stream);
pa_status pa_decode_merge(const pa_desc *desc, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *block_table,
                          const int32_t *context_lens, float scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream);

/* pa_decode in one launch (single-pass merge): the same inputs, output and
 * workspace as pa_decode, but no merge grid.  Each piece of a split
 * (sequence, kv head) writes its normalised partial rows and log-sum-exps, then
 * counts itself in at the segment's arrival counter in the workspace; the last
 * piece to arrive merges the segment's rows with the same log-sum-exp
 * arithmetic as pa_decode_merge (page "cidian.kuaisou.com: flash decoding ++":
 * the per-block results are rescaled and combined once, at the end).
 *
 * The counters are tagged with a per-call epoch, so a workspace needs no
 * clearing, and the last arrival resets its counter, so a call captured in a
 * CUDA graph may be replayed.  The result equals pa_decode's up to the order of
 * the merge's fp32 sums (the pieces are the same), and repeated calls on the
 * same inputs are bitwise identical.  Two calls in flight at once must not share
 * a workspace.  Errors as pa_decode.  A piece whose wait timed out
 * (PA_ERR_TIMEOUT) still counts itself in, so every counter returns to zero
 * even then and a captured graph may be replayed after the error is cleared. */
pa_status pa_decode_fused(const pa_desc *desc, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *block_table,
                          const int32_t *context_lens, float scale, void *out, void *workspace,
                          size_t workspace_bytes, void *stream);

size_t pa_mla_workspace_size(const pa_mla_desc *desc);

pa_status pa_decode_mla(const pa_mla_desc *desc, const void *q, const void *latent_cache,
                        const int32_t *block_table, const int32_t *context_lens, float scale,
                        void *out, void *workspace, size_t workspace_bytes, void *stream);
pa_status pa_decode_mla_partition(const pa_mla_desc *desc, const void *q,
                                  const void *latent_cache, const int32_t *block_table,
                                  const int32_t *context_lens, float scale, void *out,
                                  void *workspace, size_t workspace_bytes, void *stream);
pa_status pa_decode_mla_merge(const pa_mla_desc *desc, const void *q, const void *latent_cache,
                              const int32_t *block_table, const int32_t *context_lens,
                              float scale, void *out, void *workspace, size_t workspace_bytes,
                              void *stream);

/* pa_decode over a float8 KV cache (next step after the 16-bit path: the pages
 * name FP8 only as a Hopper capability, page "bjpcjp.github.io: llms-attention",
 * FlashAttention-3 teaser; the encoding is the OCP 8-bit float E4M3: 1 sign, 4
 * exponent bits with bias 7, 3 fraction bits, no infinity, NaN = 0x7F / 0xFF).
 *
 * k_cache / v_cache: E4M3 codes, one byte each, in the layout of pa_decode
 * ([num_blocks][num_kv_heads][block_size][head_dim]); the key is code x k_scale,
 * the value code x v_scale (one scale per tensor, finite).  q and out are
 * desc->dtype (PA_F16 or PA_BF16); the kernel computes in fp16, which holds every
 * E4M3 value exactly, so a bf16 q must lie within the fp16 range (|q| < 65504).
 * Supported: head_dim 128, and everything pa_decode supports otherwise.  The
 * workspace is sized by pa_workspace_size(desc).  Errors as pa_decode. */
pa_status pa_decode_kv_e4m3(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *context_lens, float scale, float k_scale,
                            float v_scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream);
/* Its two passes on their own, as pa_decode_partition / pa_decode_merge: the
 * merge must follow the partition pass on the same stream with the same
 * arguments and workspace. */
pa_status pa_decode_kv_e4m3_partition(const pa_desc *desc, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_table,
                                      const int32_t *context_lens, float scale, float k_scale,
                                      float v_scale, void *out, void *workspace,
                                      size_t workspace_bytes, void *stream);
pa_status pa_decode_kv_e4m3_merge(const pa_desc *desc, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_table,
                                  const int32_t *context_lens, float scale, float k_scale,
                                  float v_scale, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* Index-list decode: each sequence attends over a given list of its token
 * positions instead of [0, context length), the dense kernel behind sparse
 * attention that keeps selected entries (page "bjpcjp.github.io: llms-attention",
 * DeepSeek-V4 explainer: keep the top 1024 entries plus a sliding window, then
 * attend over them).  The selection is an input.
 *
 * token_index: device int32 [batch][max_sel]; entry i < n_sel[b] is a token
 *   position of sequence b (its K/V row is row pos % block_size of block
 *   block_table[b][pos / block_size]); entries past n_sel[b] are never read, a
 *   position listed twice counts twice, the order does not matter.
 * n_sel: device int32 [batch], 0 <= n_sel[b] <= max_sel (0 = all-zero output).
 * max_sel >= 1, with batch x (max_sel / 16 + 1) x num_kv_heads < 2^31
 * (PA_ERR_UNSUPPORTED otherwise).
 * Everything else as pa_decode (16-bit q / caches / out, head_dim 128).  A
 * position outside [0, max_blocks_per_seq x block_size) or a block id outside
 * the pool is skipped and reported as PA_ERR_BAD_BLOCK_ID by pa_device_status.
 * The workspace is sized by pa_workspace_size(desc). */
pa_status pa_decode_indexed(const pa_desc *desc, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table,
                            const int32_t *token_index, int max_sel, const int32_t *n_sel,
                            float scale, void *out, void *workspace, size_t workspace_bytes,
                            void *stream);
/* Its two passes on their own (the merge follows the partition pass on the same
 * stream with the same arguments and workspace). */
pa_status pa_decode_indexed_partition(const pa_desc *desc, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *block_table,
                                      const int32_t *token_index, int max_sel,
                                      const int32_t *n_sel, float scale, void *out,
                                      void *workspace, size_t workspace_bytes, void *stream);
pa_status pa_decode_indexed_merge(const pa_desc *desc, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_table,
                                  const int32_t *token_index, int max_sel, const int32_t *n_sel,
                                  float scale, void *out, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* Number of partitions (CTAs of the partition pass; each runs 8 independently
 * streaming warps, one piece each; 12 for the float8 and index-list paths at up to 8
 * heads per group) a call with num_partitions == 0 uses on the current
 * device (SM count x resident CTAs per SM), or -1 without a usable device.
 * kind: 0 = GQA with this head_dim, 1 = MLA (head_dim ignored), 2 = GQA over a
 * float8 KV cache (head_dim 128), 3 = index-list decode (head_dim 128). */
int pa_default_partitions(int kind, int head_dim);

/* Synchronises `stream`, then returns the first error the kernels recorded on the
 * current device since the last reset (PA_OK if none); reset != 0 clears it. */
pa_status pa_device_status(void *stream, int reset);

/* Test hook for the kernels' timeout path (not for production use).  Sets a
 * flag in device memory of the current device (a synchronous copy: call it
 * between launches).  While it is set, one warp of every partition pass that
 * runs (GQA: warp 0 of CTA 0; MLA: the copy-issuing warp of CTA 0) waits on an
 * mbarrier that nothing completes before it issues any copy; its bounded wait
 * gives up after about one second, records PA_ERR_TIMEOUT (readable through
 * pa_device_status) and the CTA finishes without it, so the call's output is
 * incomplete but the CUDA context stays usable.  The kernels read the flag when
 * they run, so a launch captured in a CUDA graph follows the flag's value at
 * replay time.  enable = 0 restores normal operation. */
void pa_test_inject_stall(int enable);

/* pa_decode without a workspace argument, for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is an integration aid.
 *
 * Some callers cannot provide scratch: a host runtime that owns all device
 * memory and lends none to plugins, a serving loop that must never call
 * cudaMalloc (it can synchronise the device and stall every stream), or a C
 * program without a caching allocator.  This entry point takes the same inputs
 * and output as pa_decode and runs the same kernels, but its scratch is a
 * fixed buffer inside the library: a file-scope device array of
 * PA_STATIC_SCRATCH_BYTES (16 MiB), present on every GPU that loads the library
 * until the process exits.  The library allocates nothing here.
 *
 *   - The first call on each device looks up the buffer's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  Later calls reuse the address.  The address
 *     belongs to the CUDA context it was looked up in: after a device reset
 *     (cudaDeviceReset) or under another context, the next call looks it up
 *     again, and that call too should come before any stream capture.
 *   - A call whose workspace (pa_workspace_size) exceeds the buffer returns
 *     PA_ERR_TOO_LARGE before launching anything.
 *   - All calls on a device share the one buffer, and it keeps the last call's
 *     contents.  Nothing in it has to start at zero, so it is never cleared.
 *     Calls that overlap on the GPU (several streams, or several host threads)
 *     race on the buffer and corrupt each other's results: serialise them.
 *   - Errors and asynchrony are as for pa_decode. */
#define PA_STATIC_SCRATCH_BYTES (16u << 20)
pa_status pa_decode_static(const pa_desc *desc, const void *q, const void *k_cache,
                           const void *v_cache, const int32_t *block_table,
                           const int32_t *context_lens, float scale, void *out, void *stream);

/* Static description of a status code. */
const char *pa_status_string(pa_status status);

#ifdef __cplusplus
}
#endif

#endif /* PA_B200_H */
