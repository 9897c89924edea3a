// Kernel parameter blocks and launchers of libsas (internal; the public ABI is include/sas.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sas {

// Radix digits of the 32-bit score keys used by the selection: 13 + 10 + 9 bits.  The score
// kernel histograms the first digit of every (b, h).
constexpr int kHistShift = 19;
constexpr int kHistBins = 1 << (32 - kHistShift);  // 8192
constexpr int kDigit2Bits = 10;
constexpr int kDigit3Bits = 9;

// ---------------------------------------------------------------------------- projection
struct ProjParams {
  const __nv_bfloat16* K;      // build: cache (layout below); append: K_new [B][Hkv][d]
  const float* M;              // [Hkv][r][d]
  void* Kproj;                 // cache layout, width r: bf16 values or FP8 E4M3 codes
  int fp8;                     // 1: write FP8 codes of (sum / kproj_scale[h])
  const float* kproj_scale;    // [Hkv] (FP8)
  const int32_t* page_table;   // [B][max_pages] or null (contiguous)
  const int32_t* seqlens;      // [B]
  uint32_t* err;               // device error word or null
  int B, Hkv, d, r, cap, max_pages, num_pages;
  int paged;                   // 0 / 1 (64-token pages)
  int append;                  // 0: build rows [0, N_b); 1: project K_new into row N_b - 1
  int rows_per_cta;            // build: rows of one (b, h) handled by one CTA
};
cudaError_t launch_proj(const ProjParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------- score scan
struct ScoreParams {
  const __nv_bfloat16* q;      // [B][Hq][d]
  const float* M;              // [Hkv][r][d]
  const void* kproj;           // cache layout, width r: bf16 values or FP8 E4M3 codes
  int fp8;                     // 1: FP8 codes, scored as kproj_scale[h] * code
  const float* kproj_scale;    // [Hkv] (FP8)
  const int32_t* page_table;
  const int32_t* seqlens;
  const int32_t* kvec;         // [B]
  const float* log_g;          // [B][Hkv][cap] or null
  uint32_t* keys;              // workspace: [B][Hkv][cap] order-preserving keys of u_i
  uint32_t* hist;              // workspace: [B][Hkv][kHistBins] counts of the keys' first digit (zero on entry)
  float* scores_out;           // [B][Hkv][cap] or null
  uint32_t* err;
  int B, Hq, Hkv, G, d, r, cap, max_pages, num_pages, paged, k_max;
  float sigma, lam;
  int ctas;                    // persistent grid size
};
void plan_score(ScoreParams& p, int num_sms);
cudaError_t launch_score(const ScoreParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------- selection
struct SelectParams {
  const uint32_t* keys;        // workspace keys written by the score kernel
  uint32_t* hist;              // workspace histograms (cleared here after use)
  const int32_t* seqlens;
  const int32_t* kvec;         // [B]
  int32_t* idx_out;            // [B][Hkv][k_max]
  uint32_t* err;
  int B, Hkv, cap, k_max;
  int cluster;                 // CTAs per (b, h)
  int threads;                 // threads per CTA (512 or 1024)
  int chunk;                   // max positions per CTA (multiple of 512)
  int cand_cap;                // candidate list capacity per CTA
  int off_hist, off_ctl, smem_bytes;
};
// Chooses cluster size and chunk for a shape; returns false if unsupported.
bool plan_select(SelectParams& p, int num_sms);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------- gather (foil)
struct GatherParams {
  const __nv_bfloat16* K;      // cache layout
  const __nv_bfloat16* V;
  const int32_t* page_table;
  const int32_t* seqlens;
  const int32_t* idx;          // [B][Hkv][k_max]
  const int32_t* kvec;         // [B]
  __nv_bfloat16* Kg;           // [B][Hkv][k_max][d]
  __nv_bfloat16* Vg;
  int32_t* counts;             // [B]
  int B, Hkv, d, cap, max_pages, num_pages, paged, k_max;
};
cudaError_t launch_gather(const GatherParams& p, cudaStream_t stream);

// ---------------------------------------------------------------------------- attention
struct AttendParams {
  const __nv_bfloat16* q;      // [B][Hq][d]
  const __nv_bfloat16* K;      // cache layout
  const __nv_bfloat16* V;
  const int32_t* page_table;
  const int32_t* seqlens;
  const int32_t* idx;          // [B][Hkv][k_max]; null for the dense (all positions) variant
  const int32_t* kvec;         // [B]; null for dense
  const float* log_g;          // [B][Hkv][cap] or null
  float* out;                  // [B][Hq][d]
  float* partials;             // workspace: [B*Hkv*ngz][splits][gt][d + 2]
  uint32_t* err;
  int B, Hq, Hkv, G, d, cap, max_pages, num_pages, paged, k_max;
  float sigma, lam;
  int gt;                      // query heads per CTA (1, 2 or 4)
  int ngz;                     // G / gt
  int splits;                  // CTAs per (b, h, head group)
  int split_len;               // index-list entries per CTA (multiple of 32)
  int max_splits;              // splits the workspace holds partials for (>= splits)
  int smem_bytes;
  int sms;                     // SMs of the device (launch-time re-split)
};
// Split plan for `count_max` index entries per head (dense: every cached row); a pure function
// of the arguments, which sizes the workspace.  launch_attend may re-split the work (up to
// max_splits) to fill whole waves of the device it runs on.
void plan_attend(AttendParams& p, int count_max, bool dense);
size_t attend_workspace_floats(const AttendParams& p);
cudaError_t launch_attend(const AttendParams& p, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit (and allows non-portable cluster sizes) on the
// current device once, not on every launch; thread-safe.
cudaError_t prepare_kernel(const void* kern, int smem_bytes, bool nonportable_cluster = false);
// Resident CTAs per SM of a kernel at a block size and dynamic shared memory (cached per device).
int ctas_per_sm(const void* kern, int threads, int smem_bytes);

// Launches kern(p) with programmatic dependent launch allowed (the kernel's pdl_wait() orders
// it after the previous kernel on the stream) and, if cluster > 0, that cluster size along x.
template <typename P>
inline cudaError_t launch_pdl(void (*kern)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, const P& p,
                              unsigned cluster = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

constexpr int kTargetCtas = 1024;       // attention split planning target (device independent)
constexpr int kMaxSplitLen = 512;       // sparse: index entries per attention CTA at most
constexpr int kMaxSplitLenDense = 2048; // dense: rows per attention CTA at most
constexpr int kMinSplitLen = 128;
constexpr int kMaxSplitsPerHead = 64;   // re-split bound (workspace partials)
constexpr int kMaxChunk = 16384;    // positions per selection CTA at most
constexpr int kMaxCluster = 16;

}  // namespace sas
