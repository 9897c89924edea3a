// Projected score scan (sm_100a): the bandwidth-bound half of the selection.
//
// JSSA page, section 打分误差的定义: the selection score of cached token i under KV head h is
// s-hat_i = q-bar^T M^T (M k_i) = q-hat . Kproj_i, with q-bar the mean of the G query heads of
// h; section Triton 内核的三个设计点: scoring is not sparse, it scans every candidate.  The gate
// of the SAS page (section 2.1) adds lambda * log g_i.  Each score is kept as the order-preserving
// uint32 key of u_i = sigma * s-hat_i (+ lambda log g_i); a per-(b, h) histogram of the keys' top
// 11 bits is accumulated for the selection that follows.
//
// The projected cache is streamed with fully coalesced 16-byte loads (a warp reads 32 rows as
// one 2*r*32-byte run per instruction group, the next batch prefetched into registers), at
// high occupancy; the keys go to the workspace with an L2 evict-last hint so that the
// selection kernel finds them on chip, the cache rows with evict-first.
#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 32;  // rows per warp per batch
constexpr int kBins = 2048;
constexpr int kMaxRowsPerCta = 64 * kWarps * kBatch;

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ldg_hint(const void* ptr, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr), "l"(pol));
  return v;
}
__device__ __forceinline__ void stg_hint(uint32_t* ptr, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.u32 [%0], %1, %2;" ::"l"(ptr), "r"(v), "l"(pol) : "memory");
}

// Warp-aggregated shared-memory histogram increment.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

template <int R, int D>
__global__ void __launch_bounds__(kThreads) score_kernel(const ScoreParams p) {
  constexpr int LPR = R / 8;         // lanes per row (16 bytes each)
  constexpr int RPI = 32 / LPR;      // rows per load instruction
  constexpr int NI = kBatch / RPI;   // load instructions per batch
  __shared__ float qbar[D];
  __shared__ float qhat[R];
  __shared__ uint32_t hist[kBins];
  __shared__ int pages_s[kMaxRowsPerCta / 64];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (blockIdx.x == 0 && tid == 0 && h == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    n = 0;
  }
  int kb = p.kvec[b];
  if (kb > p.k_max) {
    if (blockIdx.x == 0 && tid == 0 && h == 0) record_error(p.err, kDevKOverMax, (uint32_t)b);
    kb = p.k_max;
  }
  // Nothing to rank (empty selection or every position selected): no scores are needed,
  // unless the caller asked for them.  The CTA-uniform exits are expressed as one guard
  // around the body rather than early returns.
  const bool need_hist = seq_selection(kb, n).ranked;  // the selection ranks this (b, h)
  const int r0 = blockIdx.x * p.rows_per_cta;
  const int r1 = min(r0 + p.rows_per_cta, n);
  const bool skip = (!need_hist && p.scores_out == nullptr) || r0 >= r1;
  if (!skip) {
  if (p.paged) {
    for (int t = tid; t < (r1 - r0 + 63) / 64; t += kThreads) {
      int pg = p.page_table[(size_t)b * p.max_pages + r0 / 64 + t];
      if (pg < 0 || pg >= p.num_pages) {
        record_error(p.err, kDevBadPage, (uint32_t)b);
        pg = 0;
      }
      pages_s[t] = pg;
    }
  }

  // ---- q-hat = sigma * M[h] q-bar (independent vector loads) ----
  constexpr int TPR = kThreads / R;
  constexpr int CH = D / TPR;
  const int qj = tid / TPR, qpart = tid % TPR;
  float4 mreg[CH / 4];
  {
    const float4* Mrow = reinterpret_cast<const float4*>(p.M + ((size_t)h * R + qj) * D + qpart * CH);
#pragma unroll
    for (int i = 0; i < CH / 4; ++i) mreg[i] = Mrow[i];
  }
  if (tid < D) {
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + (size_t)h * p.G) * D + tid;
    float sq = 0.f;
#pragma unroll 4
    for (int g = 0; g < p.G; ++g) sq += __bfloat162float(qg[(size_t)g * D]);
    qbar[tid] = sq / (float)p.G;
  }
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  {
    float sp = 0.f;
#pragma unroll
    for (int i = 0; i < CH / 4; ++i) {
      const float* qb = qbar + qpart * CH + 4 * i;
      sp = fmaf(mreg[i].x, qb[0], sp);
      sp = fmaf(mreg[i].y, qb[1], sp);
      sp = fmaf(mreg[i].z, qb[2], sp);
      sp = fmaf(mreg[i].w, qb[3], sp);
    }
#pragma unroll
    for (int o = TPR / 2; o; o >>= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
    if (qpart == 0) qhat[qj] = sp * p.sigma;
  }
  __syncthreads();

  // This lane's 8 channels of every row it loads: chunk `part` of the row.
  const int part = lane % LPR;
  const int rsub = lane / LPR;
  float2 qv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) qv[e] = make_float2(qhat[part * 8 + 2 * e], qhat[part * 8 + 2 * e + 1]);

  const uint64_t pol_stream = policy_evict_first();
  const uint64_t pol_keep = policy_evict_last();
  const bool gated = p.log_g != nullptr;
  const size_t key_base = (size_t)bh * p.cap;

  // Address of row `pos` of this (b, h) in the projected cache.
  auto row_ptr = [&](int pos) -> const unsigned char* {
    size_t row;
    if (p.paged) {
      row = ((size_t)pages_s[(pos - r0) >> 6] * p.Hkv + h) * 64 + (pos & 63);
    } else {
      row = (size_t)bh * p.cap + pos;
    }
    return reinterpret_cast<const unsigned char*>(p.kproj + row * R);
  };

  const int nbatch = (r1 - r0 + kBatch - 1) / kBatch;
  // Batch t of this warp covers rows r0 + (warp + t*kWarps) * 32 .. +31.
  auto load = [&](int t, uint4* buf) {
    const int base = r0 + (warp + t * kWarps) * kBatch;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int pos = base + i * RPI + rsub;
      if (pos < r1) buf[i] = ldg_hint(row_ptr(pos) + part * 16, pol_stream);
      else buf[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  };

  const int my_batches = nbatch > warp ? (nbatch - warp + kWarps - 1) / kWarps : 0;
  uint4 cur[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) cur[i] = make_uint4(0u, 0u, 0u, 0u);
  if (my_batches > 0) load(0, cur);
  for (int t = 0; t < my_batches; ++t) {
    // every element of the prefetch buffer is written on every path (no read of an
    // uninitialised value on a warp's last batch)
    uint4 nxt[NI];
    if (t + 1 < my_batches) {
      load(t + 1, nxt);
    } else {
#pragma unroll
      for (int i = 0; i < NI; ++i) nxt[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    const int base = r0 + (warp + t * kWarps) * kBatch;
    // scores of rows base + i*RPI + rsub, reduced over the LPR lanes of each row
    float sc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const uint4 w = cur[i];
      float2 a = ffma2(qv[0], make_float2(bf16lo(w.x), bf16hi(w.x)), make_float2(0.f, 0.f));
      a = ffma2(qv[1], make_float2(bf16lo(w.y), bf16hi(w.y)), a);
      a = ffma2(qv[2], make_float2(bf16lo(w.z), bf16hi(w.z)), a);
      a = ffma2(qv[3], make_float2(bf16lo(w.w), bf16hi(w.w)), a);
      float s = a.x + a.y;
#pragma unroll
      for (int o = 1; o < LPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      sc[i] = s;
    }
    // lane j takes row base + j: instruction j / RPI, row slot j % RPI (held by lane slot*LPR)
    float u = 0.f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const float v = __shfl_sync(0xffffffffu, sc[i], (lane % RPI) * LPR);
      if (lane / RPI == i) u = v;
    }
    const int pos = base + lane;
    const bool valid = pos < r1;
    if (valid && gated) u = fmaf(p.lam, p.log_g[key_base + pos], u);
    const uint32_t key = float_key(u);
    if (valid) {
      stg_hint(p.keys + key_base + pos, key, pol_keep);
      if (p.scores_out != nullptr) p.scores_out[key_base + pos] = u;
    }
    hist_add(hist, key >> 21, valid);
#pragma unroll
    for (int i = 0; i < NI; ++i) cur[i] = nxt[i];
  }
  __syncthreads();
  if (need_hist) {
    uint32_t* gh = p.hist + (size_t)bh * kBins;
    for (int i = tid; i < kBins; i += kThreads) {
      const uint32_t v = hist[i];
      if (v) atomicAdd(&gh[i], v);
    }
  }
  }  // !skip
}

template <int R, int D>
cudaError_t launch_rd(const ScoreParams& p, cudaStream_t stream) {
  dim3 grid((unsigned)((p.cap + p.rows_per_cta - 1) / p.rows_per_cta), (unsigned)(p.B * p.Hkv), 1);
  score_kernel<R, D><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

void plan_score(ScoreParams& p, int num_sms) {
  // About four waves of four CTAs per SM; a whole number of warp batches per CTA.
  const long rows = (long)p.B * p.Hkv * p.cap;
  long per = rows / (16L * num_sms);
  const long unit = (long)kWarps * kBatch;
  per = (per + unit - 1) / unit * unit;
  if (per < 4 * unit) per = 4 * unit;
  if (per > kMaxRowsPerCta) per = kMaxRowsPerCta;
  p.rows_per_cta = (int)per;
}

cudaError_t launch_score(const ScoreParams& p, cudaStream_t stream) {
  if (p.d == 128) {
    switch (p.r) {
      case 16: return launch_rd<16, 128>(p, stream);
      case 32: return launch_rd<32, 128>(p, stream);
      case 64: return launch_rd<64, 128>(p, stream);
    }
  } else if (p.d == 64) {
    switch (p.r) {
      case 16: return launch_rd<16, 64>(p, stream);
      case 32: return launch_rd<32, 64>(p, stream);
      case 64: return launch_rd<64, 64>(p, stream);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace sas
