/*
 * sas.h -- C ABI of libsas: one decode step of top-k token-level sparse attention under GQA
 * on NVIDIA B200 (sm_100a).
 *
 * The method (JSSA explainer page, "JSSA 完全拆解：联合 query-key 子空间打分与 gather-free
 * 内核，训练无关的 token 级稀疏解码", pinghaoyang.com.cn):
 *   for every KV head h of sequence b, the G query heads of h are averaged into q-bar
 *   (section 打分误差的定义); every cached token i is scored on the low-rank projected key
 *   cache, s-hat_i = (M q-bar) . Kproj_i with Kproj = K M^T and M M^T = I_r (sections
 *   打分误差的定义 and 投影打分缓存与校准成本); an optional gate adds lambda * log g_i
 *   to the logit (SAS explainer page, "SAS：用门控稀疏注意力把"上下文排序"端到端对齐 LM
 *   损失", section 2.1); the top-k positions are chosen per KV head and shared by its G
 *   query heads (section JSSA 的整体结构, Figure 1); and exact softmax attention over the
 *   raw full-dimension bf16 K/V rows at those positions is computed in place, with no gather
 *   copy (section 原理详解(二) / Triton 内核的三个设计点).
 *
 * Conventions (all entry points):
 *   - Every tensor argument is a DEVICE pointer to caller-owned memory, except where stated.
 *     The library allocates nothing and never synchronises the host, except
 *     sas_check_workspace, which is a debugging aid.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     All work is enqueued on it; calls return before the GPU finishes.
 *   - Layouts are dense and row-major, in the element types stated.  bf16 is IEEE-style
 *     bfloat16.  Pointers must be 16-byte aligned.
 *   - Query head hq belongs to KV head hq / G, G = Hq / Hkv (contiguous groups).
 *   - The softmax scale is sigma = 1/sqrt(d) on attention logits and on selection scores.
 *   - Cache layouts:
 *       contiguous (page_size == 0): K, V [B][Hkv][n_cap][d] bf16; Kproj [B][Hkv][n_cap][r];
 *       paged (page_size == 64):     K, V [num_pages][Hkv][64][d] bf16;
 *                                    Kproj [num_pages][Hkv][64][r];
 *                                    page_table [B][max_pages] int32, logical token t of
 *                                    sequence b lives in page page_table[b][t / 64], row t % 64.
 *     Kproj elements are bf16 or FP8 E4M3 codes (shape.kproj_dtype).
 *     The logical capacity is cap = n_cap (contiguous) or max_pages * 64 (paged).
 *   - seqlens [B] int32: cached tokens N_b of each sequence (0 <= N_b <= cap).
 *   - Host-side validation rejects bad shapes, null or misaligned pointers and unsupported
 *     sizes with SAS_ERR_INVALID_ARG / SAS_ERR_UNSUPPORTED before anything is launched.
 *     Values the host cannot see (seqlens, page ids, k, indices) are checked on the device:
 *     a bad value sets the workspace error word (read it with sas_check_workspace), and the
 *     affected work is skipped or clamped; no kernel traps or hangs.
 *   - Launch failures return SAS_ERR_CUDA (no synchronisation is done to detect them).
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SAS_ABI_VERSION 2

typedef enum {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = 1,
  SAS_ERR_UNSUPPORTED = 2,
  SAS_ERR_CUDA = 3,
  SAS_ERR_DEVICE_CHECK = 4
} sas_status;

/* Storage type of the projected cache.
 *   SAS_KPROJ_BF16      bfloat16 values (2 bytes per element).
 *   SAS_KPROJ_FP8_E4M3  FP8 E4M3 codes (1 byte per element) with a per-KV-head fp32 scale:
 *                       the value scored is kproj_scale[h] * code (JSSA page, section
 *                       FP8 打分缓存的影响可以忽略: the scoring cache is kept in FP8).  Codes
 *                       are produced by rounding to nearest even and saturating at +-448. */
typedef enum { SAS_KPROJ_BF16 = 0, SAS_KPROJ_FP8_E4M3 = 1 } sas_kproj_dtype;

/* Problem shape shared by every call.
 *   B       sequences in the batch
 *   Hq      query heads; Hkv KV heads; Hq % Hkv == 0
 *   d       head dimension: 64 or 128
 *   r       projection rank: 16, 32 or 64, r <= d
 *   n_cap   contiguous layout: rows per (sequence, KV head) slot, a multiple of 4; 0 if paged
 *   page_size 0 (contiguous) or 64 (paged)
 *   max_pages paged: columns of the page table; num_pages: physical pages in K/V/Kproj
 *   kproj_dtype SAS_KPROJ_BF16 or SAS_KPROJ_FP8_E4M3
 *   kproj_scale device fp32 [Hkv]: the per-KV-head scale of an FP8 projected cache (read by the
 *           projection and scoring kernels); NULL for bf16.  Powers of two keep the projection's
 *           division by the scale exact; other values are divided in fp32, rounded to nearest.
 */
typedef struct {
  int32_t B, Hq, Hkv, d, r;
  int32_t n_cap;
  int32_t page_size;
  int32_t max_pages;
  int32_t num_pages;
  int32_t kproj_dtype;
  const float* kproj_scale;
} sas_shape;

/* Longest logical capacity (tokens per sequence) the selection kernel holds on chip. */
#define SAS_MAX_CAPACITY 262144

int sas_abi_version(void);

/* Human-readable name of a status code (static string). */
const char* sas_status_string(sas_status s);

/* Detail of the last SAS_ERR_INVALID_ARG / SAS_ERR_UNSUPPORTED / SAS_ERR_CUDA returned on the
 * calling host thread (static thread-local string; empty if none). */
const char* sas_last_error_detail(void);

/* Workspace sizes (host-only, pure functions of the arguments; 0 if the shape is invalid).
 * sas_decode_workspace_bytes covers sas_decode_step, sas_select_topk and
 * sas_sparse_attention with budget bound k_max; sas_dense_workspace_bytes covers
 * sas_dense_decode. */
size_t sas_decode_workspace_bytes(const sas_shape* shape, int32_t k_max);
size_t sas_dense_workspace_bytes(const sas_shape* shape);

/* Zero a workspace.  Must be called once after the workspace is allocated (or any time
 * after a call was abandoned); the kernels leave it ready for the next call themselves.
 * Enqueued on `stream`. */
sas_status sas_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Debugging aid (synchronises `stream`): copies the device error word to *code_out (0 if no
 * device-side check failed since the last init/check; see sas_device.cuh codes 1..5), the
 * batch index or position it concerns to *where_out (may be NULL), clears it, and returns
 * SAS_ERR_DEVICE_CHECK if it was set, else SAS_OK. */
sas_status sas_check_workspace(void* workspace, size_t ws_bytes, void* stream,
                               uint32_t* code_out, uint32_t* where_out);

/* Projected score cache, built over the whole cache (prefill).
 *   Kproj[b,h,i,:] = bf16_rn( sum_c K[b,h,i,c] * M[h,:,c] ), fp32 accumulation, for i < N_b;
 *   FP8: e4m3_rn_satfinite( that fp32 sum / kproj_scale[h] ).
 *   K    bf16 cache (layout above), read;  M fp32 [Hkv][r][d] orthonormal rows, read;
 *   Kproj bf16 (same layout family as K, width r), rows i < N_b written, others untouched;
 *   page_table NULL for the contiguous layout.
 * (JSSA page, section 投影打分缓存与校准成本: Kproj = K M^T, an auxiliary cache used only for
 * selection.) */
sas_status sas_build_proj_cache(const sas_shape* shape, const void* K, const float* M, void* Kproj,
                                const int32_t* page_table, const int32_t* seqlens, void* stream);

/* Projection-and-append of the newest key of every sequence, once per decode step.
 *   K_new bf16 [B][Hkv][d]: the key just produced for position N_b - 1 (seqlens already
 *   count it).  Writes Kproj at logical position N_b - 1 of every (b, h); sequences with
 *   N_b == 0 are skipped.
 * (JSSA page, section 组件级拆解 / Figure 9: the key projection is the cheapest phase.) */
sas_status sas_append_proj(const sas_shape* shape, const void* K_new, const float* M, void* Kproj,
                           const int32_t* page_table, const int32_t* seqlens, void* stream);

/* One sparse decode step: group-mean query -> projected scores (+ gate) -> per-KV-head top-k
 * -> gather-free split-K attention -> combine.
 *   q        bf16 [B][Hq][d]
 *   M        fp32 [Hkv][r][d], the scoring basis (orthonormal rows), read
 *   Kproj, K, V, page_table, seqlens: caches as above (read)
 *   k        int32 [B] (device): budget k_b; the selected set has min(k_b, N_b) positions
 *            (k_b <= 0 or N_b == 0 selects nothing and gives a zero output row);
 *            k_b > k_max is clamped to k_max and flagged in the error word
 *   k_max    host bound on k_b, >= 1; sizes idx_out and the workspace
 *   lambda   gate weight; 0 disables the gate (log_g is then not read and may be NULL)
 *   log_g    fp32 [B][Hkv][cap] (device), log g_i by logical position, finite, read when
 *            lambda != 0; u_i = sigma * s-hat_i + lambda * log g_i is the selection key and
 *            z_i = sigma * q . K_i + lambda * log g_i the attention logit
 *   out      fp32 [B][Hq][d], written
 *   idx_out  int32 [B][Hkv][k_max], written: the selected positions of each (b, h) in
 *            ascending order, padded with -1.  Ties on the fp32 selection key go to the
 *            lower position.
 *   workspace device scratch of >= sas_decode_workspace_bytes(shape, k_max) bytes,
 *            initialised once with sas_workspace_init.  Calls that share a workspace must be
 *            stream-ordered.
 */
sas_status sas_decode_step(const sas_shape* shape, const void* q, const float* M, const void* Kproj,
                           const void* K, const void* V, const int32_t* page_table,
                           const int32_t* seqlens, const int32_t* k, int32_t k_max, float lambda,
                           const float* log_g, float* out, int32_t* idx_out, void* workspace,
                           size_t ws_bytes, void* stream);

/* The selection half of sas_decode_step alone (score scan + top-k).  scores_out, if not NULL,
 * receives the fp32 selection keys u_i, [B][Hkv][cap] (positions >= N_b untouched); it is a
 * test and inspection aid, not part of the decode step's traffic. */
sas_status sas_select_topk(const sas_shape* shape, const void* q, const float* M, const void* Kproj,
                           const int32_t* page_table, const int32_t* seqlens, const int32_t* k,
                           int32_t k_max, float lambda, const float* log_g, int32_t* idx_out,
                           float* scores_out, void* workspace, size_t ws_bytes, void* stream);

/* The two halves of sas_select_topk, for composing or timing them separately; they share
 * the workspace (the scan leaves per-position keys and per-(b, h) histograms in it, the
 * selection consumes and clears the histograms).  Run them in this order on one stream.
 *   sas_score_scan: every cached token of every (b, h) is scored on the projected cache
 *     (JSSA page, section Triton 内核的三个设计点: scoring scans every candidate);
 *     arguments as sas_select_topk.
 *   sas_select_from_scores: the per-KV-head top-k of the scanned keys into idx_out. */
sas_status sas_score_scan(const sas_shape* shape, const void* q, const float* M, const void* Kproj,
                          const int32_t* page_table, const int32_t* seqlens, const int32_t* k,
                          int32_t k_max, float lambda, const float* log_g, float* scores_out,
                          void* workspace, size_t ws_bytes, void* stream);
sas_status sas_select_from_scores(const sas_shape* shape, const int32_t* seqlens, const int32_t* k,
                                  int32_t k_max, int32_t* idx_out, void* workspace, size_t ws_bytes,
                                  void* stream);

/* The attention half of sas_decode_step alone: softmax attention of every query head over
 * the first min(k_b, N_b) entries of its KV head's index list idx [B][Hkv][k_max] (any order,
 * entries in [0, N_b)), reading K/V rows in place. */
sas_status sas_sparse_attention(const sas_shape* shape, const void* q, const void* K, const void* V,
                                const int32_t* page_table, const int32_t* seqlens,
                                const int32_t* idx, const int32_t* k, int32_t k_max, float lambda,
                                const float* log_g, float* out, void* workspace, size_t ws_bytes,
                                void* stream);

/* Dense full-KV decode (the speed baseline): softmax attention of every query head over all
 * N_b cached rows, no gate.  out fp32 [B][Hq][d].  Workspace: sas_dense_workspace_bytes. */
sas_status sas_dense_decode(const sas_shape* shape, const void* q, const void* K, const void* V,
                            const int32_t* page_table, const int32_t* seqlens, float* out,
                            void* workspace, size_t ws_bytes, void* stream);

/* Gather of the selected rows, for measuring the gather-then-attend alternative (not part of
 * the decode step): copies the K and V rows at the first min(k_b, N_b) entries of every
 * (b, h) index list into contiguous buffers -- the staging copy a gather-based sparse
 * attention makes and sas_sparse_attention avoids (JSSA page, section gather 到底贵在哪).
 * sas_dense_decode over the gathered rows (a contiguous shape with n_cap = k_max and seqlens =
 * counts) then computes what sas_sparse_attention computes without a gate.
 *   idx     int32 [B][Hkv][k_max] (device), as written by the selection; entries outside
 *           [0, N_b) read position 0
 *   Kg, Vg  bf16 [B][Hkv][k_max][d] (device), written for the first counts[b] rows
 *   counts  int32 [B] (device), written: min(k_b, k_max, N_b)
 */
sas_status sas_gather_selected(const sas_shape* shape, const void* K, const void* V,
                               const int32_t* page_table, const int32_t* seqlens,
                               const int32_t* idx, const int32_t* k, int32_t k_max, void* Kg,
                               void* Vg, int32_t* counts, void* stream);

/* Bytes of the library's fixed scratch array (16 MiB), used by sas_decode_step_static_scratch. */
#define SAS_STATIC_SCRATCH_BYTES (16u << 20)

/* sas_decode_step without a caller workspace.  The pages describe no such call: it is an
 * interface convenience with no counterpart in the method.
 *
 * Who needs it: callers that cannot hand the library device memory, e.g. a C or C++ host
 * that owns no device allocator and must not call cudaMalloc on its decode path (cudaMalloc
 * can stall the whole device), or a plug-in inside a framework whose caching allocator owns
 * every byte of device memory and offers extension code no scratch buffer.  This call makes
 * no allocation of any kind: its scratch is a fixed array of SAS_STATIC_SCRATCH_BYTES in the
 * library's device image, placed by the CUDA driver when the library's device code is loaded
 * on a device (at its first use under lazy module loading, CUDA's default).
 *
 * Arguments, outputs and results are those of sas_decode_step (same kernels, same launch
 * configuration); there is no workspace argument.
 *
 * Size limit: the shape and k_max must need at most SAS_STATIC_SCRATCH_BYTES of workspace,
 * i.e. sas_decode_workspace_bytes(shape, k_max) <= SAS_STATIC_SCRATCH_BYTES.  For example
 * B=1, Hq=32, Hkv=8, d=128, r=32, 131072 tokens, k_max=4096 needs 4,989,184 bytes (4.8 MiB) and
 * B=4 at 65536 tokens 11,567,360 bytes (11.0 MiB); B=16 at 131072 tokens needs 79,823,104 bytes
 * (76.1 MiB) and is rejected.  A shape
 * over the limit returns SAS_ERR_UNSUPPORTED before anything is launched, with the sizes in
 * sas_last_error_detail(); use sas_decode_step with a workspace for it.
 *
 * Setup: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current, and caches it with the id of the device's
 * current CUDA context; make that first call before any stream capture begins.  If that context
 * is later replaced (cudaDeviceReset, or the primary context torn down and created again), the
 * next call looks the address up again, so it too should come before any capture.  The current
 * device selects which device's array is used.
 *
 * Sharing: all calls on one device use the same array.  Calls that overlap in time on that
 * device (different streams, or different host threads, without ordering between them) race
 * on it and give wrong results; order them on one stream.  Each call first clears, on
 * `stream`, the part of the array that must start at zero (the device error word and the
 * per-head histograms); the rest is written before it is read.
 *
 * Device-side checks still run, but their error word lives in the shared array, is cleared by
 * the next call and cannot be read with sas_check_workspace: callers that need the device
 * checks reported use sas_decode_step with their own workspace. */
sas_status sas_decode_step_static_scratch(const sas_shape* shape, const void* q, const float* M,
                                          const void* Kproj, const void* K, const void* V,
                                          const int32_t* page_table, const int32_t* seqlens,
                                          const int32_t* k, int32_t k_max, float lambda,
                                          const float* log_g, float* out, int32_t* idx_out,
                                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H_ */
