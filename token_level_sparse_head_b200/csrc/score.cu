// Projected score scan (sm_100a): the bandwidth-bound half of the selection.
//
// JSSA page, section 打分误差的定义: the selection score of cached token i under KV head h is
// s-hat_i = q-bar^T M^T (M k_i) = q-hat . Kproj_i, with q-bar the mean of the G query heads of
// h; section Triton 内核的三个设计点: scoring is not sparse, it scans every candidate.  The gate
// of the SAS page (section 2.1) adds lambda * log g_i.  Each score is turned into the
// order-preserving uint32 key of u_i = sigma * s-hat_i (+ lambda log g_i), written to the
// workspace with an L2 evict-last hint for the selection that follows, and a histogram of the
// keys' top 13 bits is accumulated per (b, h).
//
// Persistent kernel, one CTA per SM.  The work is the list of 4 KB blocks of projected rows
// (64 rows at r = 32 in bf16) of every (b, h) that needs scores, in (b, h, position) order; each
// CTA takes one contiguous, equal share of it.  A producer warp streams the blocks into a ring of
// 32 shared-memory slots with bulk copies (TMA engine, mbarrier completion); each producer lane
// owns one slot.  Sixteen consumer warps take the blocks in turn, two slots each: a consumer warp
// moves a landed block into registers (eight 16-byte pieces per lane) and hands the slot straight
// back to its producer lane before computing, so a slot is out of flight only for the few
// shared-memory loads that empty it.  Per 32-row batch the lanes form 16-byte dot products with
// q-hat and meet in a transposing butterfly.

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kBlockBytes = 4096;   // projected bytes per block (one ring stage)
constexpr int kDepth = 2;           // ring slots per consumer warp
constexpr int kMaxWarps = 16;       // consumer warps per CTA at most
constexpr int kSmemLimit = 227 * 1024;
constexpr int kSmemMisc = 2048;     // q-bar, q-hat, barriers and plan (upper bound)

// Row geometry of the projected cache: bf16 (KP8 = false) or FP8 E4M3 codes (KP8 = true).
template <int R, bool KP8>
struct Geo {
  static constexpr int ROW_BYTES = KP8 ? R : 2 * R;
  static constexpr int BLOCK_ROWS = kBlockBytes / ROW_BYTES;  // bf16: 128 / 64 / 32 for r = 16 / 32 / 64
  static constexpr int NB = BLOCK_ROWS / 32;                  // 32-row batches per block
  static constexpr int CPL = KP8 ? 16 : 8;  // channels per 16-byte load
  static constexpr int LPR = R / CPL;       // lanes per row
  static constexpr int RPI = 32 / LPR;      // rows per load instruction
  static constexpr int NI = LPR;            // load instructions per 32-row batch
  static constexpr int LOG_LPR = LPR == 1 ? 0 : LPR == 2 ? 1 : LPR == 4 ? 2 : 3;
};

// Block shape of one instantiation: as many consumer warps (two slots each) as shared memory
// holds next to the histogram, at most 16, and one producer lane per slot.
template <int R, bool GATED, bool KP8>
struct Cfg {
  using Gm = Geo<R, KP8>;
  static constexpr int kBins = kHistBins;
  static constexpr int kSlotBytes = kBlockBytes + (GATED ? Gm::BLOCK_ROWS * 4 : 0);
  static constexpr int kMaxSlots = (kSmemLimit - kSmemMisc - kBins * 4) / kSlotBytes;
  static constexpr int kWarps = kMaxSlots / kDepth >= kMaxWarps ? kMaxWarps : kMaxSlots / kDepth;
  static constexpr int kSlots = kWarps * kDepth;
  static constexpr int kConsumers = kWarps * 32;
  static constexpr int kProducerWarps = (kSlots + 31) / 32;
  static constexpr int kThreads = kConsumers + kProducerWarps * 32;
};

// Position of a CTA's share in the block list, computed once by warp 0.
struct Plan {
  int count;  // blocks of this CTA
  int b0;     // sequence of the first block
  int h0, c0; // KV head and block index within it
};

template <int R, int D, bool GATED, bool KP8>
struct Smem {
  using C = Cfg<R, GATED, KP8>;
  unsigned char ring[C::kSlots][C::kSlotBytes];
  uint32_t hist[C::kBins];
  float qbar[D];
  float qhat[R];
  uint64_t full[C::kSlots];
  uint64_t empty[C::kSlots];
  Plan plan;
};

template <int R, int D, bool GATED, bool KP8>
constexpr bool smem_fits() {
  return sizeof(Smem<R, D, GATED, KP8>) <= (size_t)kSmemLimit;
}
static_assert(smem_fits<16, 128, true, true>() && smem_fits<32, 128, true, true>() && smem_fits<64, 128, true, true>() &&
                  smem_fits<16, 128, true, false>() && smem_fits<32, 128, true, false>() &&
                  smem_fits<64, 128, true, false>() && smem_fits<32, 128, false, false>(),
              "score kernel shared memory");

__device__ __forceinline__ void stg_hint(uint32_t* ptr, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.u32 [%0], %1, %2;" ::"l"(ptr), "r"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Barrier 1 among the consumer warps (the producer warp never joins it).
template <int N>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

// Dot product of 8 bf16 values (one 16-byte chunk of a row) with this lane's 8 channels of q-hat.
__device__ __forceinline__ float dot8(const float2 (&qv)[4], uint4 w) {
  float2 a = ffma2(qv[0], make_float2(bf16lo(w.x), bf16hi(w.x)), make_float2(0.f, 0.f));
  a = ffma2(qv[1], make_float2(bf16lo(w.y), bf16hi(w.y)), a);
  a = ffma2(qv[2], make_float2(bf16lo(w.z), bf16hi(w.z)), a);
  a = ffma2(qv[3], make_float2(bf16lo(w.w), bf16hi(w.w)), a);
  return a.x + a.y;
}

// Dot product of 16 FP8 E4M3 codes (one 16-byte chunk of a row, code 2i in the low byte of
// each 16-bit half) with this lane's 16 channels of q-hat (already times the head's scale).
__device__ __forceinline__ float dot16_fp8(const float2 (&qv)[8], uint4 w) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  float2 a = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(ws[i] & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(ws[i] >> 16), __NV_E4M3);
    a = ffma2(qv[2 * i], __half22float2(__half2(lo)), a);
    a = ffma2(qv[2 * i + 1], __half22float2(__half2(hi)), a);
  }
  return a.x + a.y;
}

// Transposing butterfly over the LPR lanes of a row: v[i] holds this lane's partial dot of row
// i * RPI + rsub; afterwards the result is the full score of row part * RPI + rsub.
template <class Gm>
__device__ __forceinline__ float butterfly(float (&v)[Gm::NI], int lane) {
#pragma unroll
  for (int lvl = 0; lvl < Gm::LOG_LPR; ++lvl) {
    const int m = Gm::LPR >> (lvl + 1);
    const int half = Gm::NI >> (lvl + 1);
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return v[0];
}

// Cached length, budget and scored block count of one sequence.  Every warp computes the same
// values (bad inputs are recorded once, by CTA 0's plan).
struct SeqInfo {
  int n;        // N_b (0 if out of range)
  int k_eff;    // min(k_b, N_b), k_b clamped to k_max
  int blocks;   // blocks that need scores (0 when nothing is ranked or reported)
  bool ranked;  // the selection ranks this sequence
};
template <int BR>
__device__ __forceinline__ SeqInfo seq_info(const ScoreParams& p, int b, bool record) {
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (record) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    n = 0;
  }
  int kb = p.kvec[b];
  if (kb > p.k_max) {
    if (record) record_error(p.err, kDevKOverMax, (uint32_t)b);
    kb = p.k_max;
  }
  SeqInfo s;
  s.n = n;
  const SeqSelection sel = seq_selection(kb, n);
  s.k_eff = sel.k_eff;
  s.ranked = sel.ranked;
  s.blocks = (s.ranked || p.scores_out != nullptr) ? (n + BR - 1) / BR : 0;
  return s;
}

// The first (b, h) at or after sequence b with blocks to score (b == B when there is none).
template <int BR>
__device__ __forceinline__ void next_scored_seq(const ScoreParams& p, int& b, SeqInfo& si) {
  while (b < p.B && (si = seq_info<BR>(p, b, false)).blocks == 0) ++b;
}

template <int R, int D, bool GATED, bool KP8>
__global__ void __launch_bounds__(Cfg<R, GATED, KP8>::kThreads, 1) score_kernel(const ScoreParams p) {
  using C = Cfg<R, GATED, KP8>;
  using Gm = Geo<R, KP8>;
  constexpr int BR = Gm::BLOCK_ROWS;
  constexpr int NW = C::kWarps;
  constexpr int kConsumers = C::kConsumers;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem<R, D, GATED, KP8>& S = *reinterpret_cast<Smem<R, D, GATED, KP8>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    fence_barrier_init();
  }
  for (int i = tid; i < C::kBins; i += C::kThreads) S.hist[i] = 0u;

  // ---- this CTA's share of the block list (warp 0) ----
  if (warp == 0) {
    // per-lane block counts of sequences lane, lane + 32, ...; the first 32 are kept
    long long mine = 0;
    long long first = 0;
    for (int b = lane; b < p.B; b += 32) {
      const long long c = (long long)p.Hkv * seq_info<BR>(p, b, blockIdx.x == 0).blocks;
      if (b < 32) first = c;
      mine += c;
    }
    long long total = mine;
#pragma unroll
    for (int o = 16; o; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
    const long long beg = total * blockIdx.x / gridDim.x;
    const long long end = total * (blockIdx.x + 1) / gridDim.x;
    // first sequence whose blocks contain `beg`
    int b0 = p.B;
    long long before = 0, cum = 0;
    if (beg < end) {
      for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        long long cnt = first;
        if (base > 0) cnt = b < p.B ? (long long)p.Hkv * seq_info<BR>(p, b, false).blocks : 0;
        if (b >= p.B) cnt = 0;
        long long incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const long long start = cum + incl - cnt;
        const uint32_t hit = __ballot_sync(0xffffffffu, cnt > 0 && start <= beg && beg < start + cnt);
        if (hit) {
          const int l = __ffs(hit) - 1;
          b0 = base + l;
          before = __shfl_sync(0xffffffffu, start, l);
          break;
        }
        cum += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) {
      Plan pl = {0, p.B, 0, 0};
      if (b0 < p.B) {
        const int nb = seq_info<BR>(p, b0, false).blocks;
        const long long off = beg - before;
        pl.count = (int)(end - beg);
        pl.b0 = b0;
        pl.h0 = (int)(off / nb);
        pl.c0 = (int)(off % nb);
      }
      S.plan = pl;
    }
  }
  __syncthreads();
  // The projected cache (appended to by the previous kernel), the keys, the histograms and the
  // error word are touched only from here on.
  pdl_wait();
  pdl_trigger();
  const Plan pl = S.plan;

  bool waited_ok = true;
  const unsigned char* kp = reinterpret_cast<const unsigned char*>(p.kproj);

  if (warp >= NW) {
    // ---------------------------------------------------------------- producers
    // Producer lane L owns ring slot L and copies the CTA's blocks L, L + kSlots, ... into it,
    // each once the consumer warp that read the slot's previous block has released it.
    const int L = (warp - NW) * 32 + lane;
    if (L < C::kSlots && pl.count > L) {
      int b = pl.b0, h = pl.h0, c = pl.c0;
      SeqInfo si = seq_info<BR>(p, b, false);
      // move the walk k blocks forward
      auto advance = [&](int k) {
        while (k > 0 && b < p.B) {
          const int take = min(k, si.blocks - c);
          c += take;
          k -= take;
          if (c == si.blocks) {
            c = 0;
            if (++h == p.Hkv) {
              h = 0;
              ++b;
              next_scored_seq<BR>(p, b, si);
            }
          }
        }
      };
      advance(L);
      const int slot = L;
      uint32_t phase = 0u;
      for (int t = L; t < pl.count; t += C::kSlots) {
        if (t >= C::kSlots) {
          if (!mbar_wait_bounded(&S.empty[slot], phase)) waited_ok = false;
          phase ^= 1u;
        }
        const int row0 = c * BR;
        const int rows = min(BR, si.n - row0);
        const int bh = b * p.Hkv + h;
        // gate values: a whole number of 16-byte units, inside the [cap] row (cap % 4 == 0)
        const uint32_t lg_bytes = GATED ? (uint32_t)((rows + 3) & ~3) * 4u : 0u;
        unsigned char* dst = S.ring[slot];
        mbar_arrive_expect_tx(&S.full[slot], (uint32_t)rows * Gm::ROW_BYTES + lg_bytes);
        if (!p.paged) {
          bulk_g2s(dst, kp + ((size_t)bh * p.cap + row0) * Gm::ROW_BYTES, (uint32_t)rows * Gm::ROW_BYTES,
                   &S.full[slot]);
        } else {
          const int32_t* pt = p.page_table + (size_t)b * p.max_pages;
          for (int g = row0; g < row0 + rows;) {
            const int pr = min(64 - (g & 63), row0 + rows - g);  // rows in this page piece
            int pg = pt[g >> 6];
            if (pg < 0 || pg >= p.num_pages) {
              record_error(p.err, kDevBadPage, (uint32_t)b);
              pg = 0;
            }
            bulk_g2s(dst + (size_t)(g - row0) * Gm::ROW_BYTES,
                     kp + (((size_t)pg * p.Hkv + h) * 64 + (g & 63)) * Gm::ROW_BYTES, (uint32_t)pr * Gm::ROW_BYTES,
                     &S.full[slot]);
            g += pr;
          }
        }
        if (GATED) bulk_g2s(dst + kBlockBytes, p.log_g + (size_t)bh * p.cap + row0, lg_bytes, &S.full[slot]);
        advance(C::kSlots);
      }
    }
    if (!waited_ok) record_error(p.err, kDevWaitTimeout, blockIdx.x);
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  const uint64_t pol_keep = l2_evict_last();
  const int part = lane % Gm::LPR;  // this lane's 16-byte chunk of each row it loads
  const int rsub = lane / Gm::LPR;  // its row within each load instruction
  float2 qv[Gm::CPL / 2];
  int cur_bh = -1;
  bool cur_ranked = false;
  // The key of this lane's row of a 32-row batch (valid: the row is < N_b) into the keys buffer
  // and the histogram (and the fp32 score into scores_out when asked for).
  auto take_key = [&](float u, int bh, int pos, bool valid) {
    if (valid) {
      const uint32_t key = float_key(u);
      stg_hint(p.keys + (size_t)bh * p.cap + pos, key, pol_keep);
      if (cur_ranked) atomicAdd(&S.hist[key >> kHistShift], 1u);
      if (p.scores_out != nullptr) p.scores_out[(size_t)bh * p.cap + pos] = u;
    }
  };

  int b = pl.b0, h = pl.h0, c = pl.c0;
  SeqInfo si = seq_info<BR>(p, b < p.B ? b : 0, false);
  int t = 0;  // blocks of the CTA before the current head segment
  while (t < pl.count) {
    const int seg = min(si.blocks - c, pl.count - t);  // blocks of this head in the share
    const int bh = b * p.Hkv + h;
    // ---- new head (every consumer warp, whether or not it gets blocks of it) ----
    {
      // TPR threads per output of q-hat: a power of two with R * TPR <= kConsumers
      constexpr int TPR = (kConsumers / R) >= 32 ? 32 : (kConsumers / R) >= 16 ? 16 : (kConsumers / R) >= 8 ? 8 : 4;
      constexpr int CH = D / TPR;
      const int qj = tid / TPR, qpart = tid % TPR;
      const bool qrow = qj < R;
      float mreg[CH];
      const float* Mrow = p.M + ((size_t)h * R + (qrow ? qj : 0)) * D + qpart * CH;
#pragma unroll
      for (int i = 0; i < CH; ++i) mreg[i] = Mrow[i];
      consumers_sync<kConsumers>();  // every warp is done with the previous head's rows
      if (cur_bh >= 0) {
        // the previous head's counts into its global histogram, then a clear histogram
        uint32_t* gh = p.hist + (size_t)cur_bh * C::kBins;
        for (int i = tid; i < C::kBins; i += kConsumers) {
          const uint32_t v = S.hist[i];
          if (v) {
            if (cur_ranked) atomicAdd(&gh[i], v);
            S.hist[i] = 0u;
          }
        }
      }
      if (tid < D) {
        const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + (size_t)h * p.G) * D + tid;
        float sq = 0.f;
        for (int g = 0; g < p.G; ++g) sq += __bfloat162float(qg[(size_t)g * D]);
        S.qbar[tid] = sq / (float)p.G;
      }
      consumers_sync<kConsumers>();
      float sp = 0.f;
#pragma unroll
      for (int i = 0; i < CH; ++i) sp = fmaf(mreg[i], S.qbar[qpart * CH + i], sp);
#pragma unroll
      for (int o = TPR / 2; o; o >>= 1) sp += __shfl_xor_sync(0xffffffffu, sp, o);
      // FP8: the head's scale multiplies q-hat, so the codes are used as they are
      if (qpart == 0 && qrow) S.qhat[qj] = sp * p.sigma * (KP8 ? p.kproj_scale[h] : 1.f);
      consumers_sync<kConsumers>();
#pragma unroll
      for (int e = 0; e < Gm::CPL / 2; ++e)
        qv[e] = make_float2(S.qhat[part * Gm::CPL + 2 * e], S.qhat[part * Gm::CPL + 2 * e + 1]);
      cur_bh = bh;
      cur_ranked = si.ranked;
    }

    // ---- this warp's blocks of the segment: CTA block indices j = t.. with j % NW == warp ----
    const int j0 = t + ((warp - t) % NW + NW) % NW;
    for (int j = j0; j < t + seg; j += NW) {
      const int slot = j % C::kSlots;  // the warp's blocks cycle through its kDepth slots
      if (!mbar_wait_bounded(&S.full[slot], (uint32_t)(j / C::kSlots) & 1u)) waited_ok = false;
      const int row0 = (c + (j - t)) * BR;
      const int rows = min(BR, si.n - row0);
      const unsigned char* st = S.ring[slot];
      // The whole block into registers (8 16-byte pieces per lane) and the slot straight back to
      // its producer lane, so the arithmetic below overlaps the copy of the slot's next block.
      // Rows past a partial block's end hold older data; their results are dropped below.
      uint4 wv[Gm::NB][Gm::NI];
      float lgv[Gm::NB];
#pragma unroll
      for (int bt = 0; bt < Gm::NB; ++bt) {
#pragma unroll
        for (int ii = 0; ii < Gm::NI; ++ii)
          wv[bt][ii] = *reinterpret_cast<const uint4*>(st + (size_t)(bt * 32 + ii * Gm::RPI + rsub) * Gm::ROW_BYTES +
                                                       part * 16);
        if constexpr (GATED) lgv[bt] = reinterpret_cast<const float*>(st + kBlockBytes)[bt * 32 + part * Gm::RPI + rsub];
      }
      __syncwarp();  // every lane has read the slot
      if (lane == 0) mbar_arrive(&S.empty[slot]);
#pragma unroll
      for (int bt = 0; bt < Gm::NB; ++bt) {
        const int wrows = rows - bt * 32;  // rows of this 32-row batch (warp-uniform)
        if (wrows > 0) {
          float v[Gm::NI];
#pragma unroll
          for (int ii = 0; ii < Gm::NI; ++ii) {
            if constexpr (KP8) v[ii] = dot16_fp8(qv, wv[bt][ii]); else v[ii] = dot8(qv, wv[bt][ii]);
          }
          const float u0 = butterfly<Gm>(v, lane);
          const int lr = part * Gm::RPI + rsub;
          const float u = GATED ? fmaf(p.lam, lgv[bt], u0) : u0;
          take_key(u, bh, row0 + bt * 32 + lr, lr < wrows);
        }
      }
    }

    // ---- next head ----
    t += seg;
    c = 0;
    if (++h == p.Hkv) {
      h = 0;
      ++b;
      next_scored_seq<BR>(p, b, si);
    }
  }
  consumers_sync<kConsumers>();
  if (cur_bh >= 0 && cur_ranked) {
    uint32_t* gh = p.hist + (size_t)cur_bh * C::kBins;
    for (int i = tid; i < C::kBins; i += kConsumers) {
      const uint32_t v = S.hist[i];
      if (v) atomicAdd(&gh[i], v);
    }
  }
  if (!waited_ok) record_error(p.err, kDevWaitTimeout, blockIdx.x);
}

template <int R, int D, bool GATED, bool KP8>
cudaError_t launch_v(const ScoreParams& p, cudaStream_t stream) {
  using C = Cfg<R, GATED, KP8>;
  auto kern = score_kernel<R, D, GATED, KP8>;
  const int smem = (int)sizeof(Smem<R, D, GATED, KP8>);
  cudaError_t e = prepare_kernel((const void*)kern, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)p.ctas), dim3(C::kThreads), (size_t)smem, stream, p);
}

template <int R, int D>
cudaError_t launch_rd(const ScoreParams& p, cudaStream_t stream) {
  const bool gated = p.log_g != nullptr;
  if (p.fp8) return gated ? launch_v<R, D, true, true>(p, stream) : launch_v<R, D, false, true>(p, stream);
  return gated ? launch_v<R, D, true, false>(p, stream) : launch_v<R, D, false, false>(p, stream);
}

}  // namespace

void plan_score(ScoreParams& p, int num_sms) {
  // Persistent: one CTA per SM, never more CTAs than there can be blocks.
  const int br = kBlockBytes / ((p.fp8 ? 1 : 2) * p.r);
  const long long blocks = (long long)p.B * p.Hkv * ((p.cap + br - 1) / br);
  long long ctas = num_sms;
  if (ctas > blocks) ctas = blocks;
  p.ctas = (int)(ctas < 1 ? 1 : ctas);
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
