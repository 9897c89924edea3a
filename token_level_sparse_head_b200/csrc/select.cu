// Per-KV-head top-k selection over the score keys (sm_100a).
//
// JSSA page, section JSSA 的整体结构 / Figure 1: every KV head keeps the positions of its k
// largest projected scores, and its G query heads share them; section 局限与需要留意的地方:
// no sink or recent window is forced.  The score kernel has left each (b, h)'s order-preserving
// uint32 keys in the workspace (in L2) with a histogram of their top 11 bits.
//
// A cluster of C CTAs serves one (b, h) (C = 1 when there are enough heads to fill the GPU);
// each CTA owns a contiguous chunk of positions and reads its keys from L2 twice:
//   1. the histogram gives the first 11-bit digit of the k-th largest key; the chunk is read
//      once, counting keys above that digit and keeping the keys equal to it (candidates) in
//      shared memory;
//   2. the remaining 11- and 10-bit digits come from histograms of the candidates only,
//      combined over the cluster through distributed shared memory (one cluster barrier per
//      digit); a digit whose bin holds exactly the remaining count ends the search;
//   3. the chunk is read again in tiles: positions with a larger key are selected, and of those
//      equal to the threshold key the lowest positions fill the remainder (exact ties -> lower
//      position); block-wide prefix sums per tile and a cluster-wide prefix of the CTA totals
//      give every position its output slot, so the index list comes out ascending, unsorted.
#include <cooperative_groups.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace cg = cooperative_groups;

namespace sas {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;          // 11-bit digits
constexpr int kPerThread = 16;       // keys per thread per tile (four 16-byte loads)
constexpr int kTile = kThreads * kPerThread;
constexpr int kCandCap = 8192;       // candidate keys kept on chip per CTA
constexpr int kCand2Cap = 2048;      // survivors of the second digit

struct Ctl {
  uint32_t cnt1, cnt2, gt0, pad;
  uint32_t cta_gt, cta_eq, gt_before, eq_before;
};

struct Found {
  uint32_t digit, above, eq, pad;
};

struct SelSmem {
  uint32_t hl[kBins];        // this CTA's histogram
  uint32_t gh1[kBins];       // rank 0: cluster histogram of digit 2
  uint32_t gh2[kBins / 2];   // rank 0: cluster histogram of digit 3
  uint32_t cand[kCandCap];
  uint32_t cand2[kCand2Cap];
  uint32_t wsum[kWarps];
  Ctl ctl;
  Found found;
};

// Exclusive prefix sum over the block; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint32_t off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t s = wsum[w];
    off += (w < warp) ? s : 0u;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return off + x - v;
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* wsum) {
  uint32_t tot;
  block_excl_scan(v, wsum, &tot);
  return tot;
}

// Warp-aggregated shared-memory histogram increment (many lanes share few bins).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (act == 0u) return;
  if (active) {
    const uint32_t peers = __match_any_sync(act, bin);
    if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
  }
}

// Appends `key` (where take is true) to list[] through a shared counter; warp-aggregated.
__device__ __forceinline__ void list_append(uint32_t* list, uint32_t* counter, uint32_t cap, uint32_t key, bool take) {
  const uint32_t m = __ballot_sync(0xffffffffu, take);
  if (m == 0u) return;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0u;
  if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) {
    const uint32_t pos = base + (uint32_t)__popc(m & ((1u << lane) - 1u));
    if (pos < cap) list[pos] = key;
  }
}

// Digit holding the k_rem-th largest key, from a histogram of `nb` = PER * kThreads bins, read
// through a generic pointer (global memory or a cluster peer's shared memory).  Thread t covers
// digits [nb - (t+1)*PER, nb - t*PER), highest first.  Every CTA of a cluster that runs this on
// the same histogram gets the same answer.
template <int PER>
__device__ __forceinline__ void find_digit(const uint32_t* H, uint32_t k_rem, uint32_t* wsum, Found* out) {
  const int lo = PER * kThreads - ((int)threadIdx.x + 1) * PER;
  uint32_t c[PER];
  if constexpr (PER == 4) {
    const uint4 a = *reinterpret_cast<const uint4*>(H + lo);
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
  } else {
    const uint2 a = *reinterpret_cast<const uint2*>(H + lo);
    c[0] = a.x; c[1] = a.y;
  }
  uint32_t tsum = 0u;
#pragma unroll
  for (int j = 0; j < PER; ++j) tsum += c[j];
  uint32_t tot;
  const uint32_t above = block_excl_scan(tsum, wsum, &tot);
  if (above < k_rem && k_rem <= above + tsum) {
    uint32_t a = above;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j) {
      if (a + c[j] >= k_rem) {
        out->digit = (uint32_t)(lo + j);
        out->above = a;
        out->eq = c[j];
        break;
      }
      a += c[j];
    }
  }
  __syncthreads();
}

// Fire-and-forget add into the same shared-memory word of cluster CTA `rank`.
__device__ __forceinline__ void red_add_cluster(const uint32_t* local, uint32_t rank, uint32_t v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}

// Keys [t*kTile + tid*kPerThread, +kPerThread) of the chunk; positions past len read as 0 (and
// are masked by the callers).
__device__ __forceinline__ void load_tile(const uint32_t* gk, int len, int t, uint32_t (&k)[kPerThread]) {
  const int li = t * kTile + (int)threadIdx.x * kPerThread;
  if (li + kPerThread <= len) {
#pragma unroll
    for (int v = 0; v < kPerThread / 4; ++v) {
      const uint4 a = __ldcg(reinterpret_cast<const uint4*>(gk + li + 4 * v));
      k[4 * v + 0] = a.x; k[4 * v + 1] = a.y; k[4 * v + 2] = a.z; k[4 * v + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) k[e] = (li + e < len) ? __ldcg(gk + li + e) : 0u;
  }
}

__global__ void __launch_bounds__(kThreads, 2) select_topk_kernel(const SelectParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelSmem& S = *reinterpret_cast<SelSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int C = (int)cluster.num_blocks();
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;

  // per-sequence values (range errors were recorded by the score kernel)
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) n = 0;
  const SeqSelection sel = seq_selection(min(p.kvec[b], p.k_max), n);
  const int k_eff = sel.k_eff;
  int32_t* idx = p.idx_out + (size_t)bh * p.k_max;
  // Nothing to rank: empty selection, or every position selected (uniform per cluster).
  // The exits are one guard around the body, not early returns.
  const bool trivial = !sel.ranked;

  // this CTA's positions [c0, c1): chunks of whole 16-byte groups
  const int chunk_b = (((n + C - 1) / C) + 15) & ~15;
  const int c0 = min(rank * chunk_b, n);
  const int c1 = min(c0 + chunk_b, n);
  const int len = c1 - c0;
  const uint32_t* gk = p.keys + (size_t)bh * p.cap + c0;
  const int ntiles = (len + kTile - 1) / kTile;

  if (trivial) {
    for (int j = rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = (j < k_eff) ? j : -1;
  } else {
    for (int i = tid; i < kBins + kBins + kBins / 2; i += kThreads) S.hl[i] = 0u;  // hl, gh1, gh2
    if (tid == 0) {
      S.ctl.cnt1 = 0u;
      S.ctl.cnt2 = 0u;
    }
    // ---- digit 1 from the global histogram ----
    const uint32_t* ghist = p.hist + (size_t)bh * kBins;
    uint32_t k_rem = (uint32_t)k_eff;
    find_digit<4>(ghist, k_rem, S.wsum, &S.found);
    const uint32_t d0 = S.found.digit;
    uint32_t prefix = d0 << 21;
    uint32_t mask = 0x7ffu << 21;
    k_rem -= S.found.above;
    bool done = (S.found.eq == k_rem);

    // ---- pass 1 over the chunk: keys above digit 1, candidates equal to it ----
    uint32_t gt0 = 0u, eq0 = 0u;
    {
      uint32_t cur[kPerThread];
#pragma unroll
      for (int e = 0; e < kPerThread; ++e) cur[e] = 0u;
      if (ntiles > 0) load_tile(gk, len, 0, cur);
      for (int t = 0; t < ntiles; ++t) {
        uint32_t nxt[kPerThread];
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) nxt[e] = 0u;
        if (t + 1 < ntiles) load_tile(gk, len, t + 1, nxt);
        const int li = t * kTile + tid * kPerThread;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          const bool valid = li + e < len;
          const uint32_t dg = cur[e] >> 21;
          gt0 += (valid && dg > d0) ? 1u : 0u;
          eq0 += (valid && dg == d0) ? 1u : 0u;
          if (!done) list_append(S.cand, &S.ctl.cnt1, kCandCap, cur[e], valid && dg == d0);
        }
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) cur[e] = nxt[e];
      }
    }
    __syncthreads();
    // Every CTA has read the global histogram and zeroed its cluster histograms: after this
    // barrier rank 0 clears the global histogram for the next call, and the adds may start.
    if (C > 1) cluster.sync();
    if (rank == 0)
      for (int i = tid; i < kBins; i += kThreads) const_cast<uint32_t*>(ghist)[i] = 0u;

    const uint32_t n1 = S.ctl.cnt1;
    const bool ovf1 = n1 > (uint32_t)kCandCap;
    // ---- digit 2: histogram of the candidates, summed over the cluster in rank 0 ----
    if (!done) {
      if (!ovf1) {
        for (uint32_t e0 = 0; e0 < n1; e0 += kThreads) {
          const uint32_t e = e0 + tid;
          const uint32_t key = e < n1 ? S.cand[e] : 0u;
          hist_add(S.hl, (key >> 10) & 0x7ffu, e < n1);
        }
      } else {
        for (int t = 0; t < ntiles; ++t) {
          uint32_t k[kPerThread];
          load_tile(gk, len, t, k);
          const int li = t * kTile + tid * kPerThread;
#pragma unroll
          for (int e = 0; e < kPerThread; ++e)
            hist_add(S.hl, (k[e] >> 10) & 0x7ffu, li + e < len && (k[e] & mask) == prefix);
        }
      }
      __syncthreads();
      const uint32_t* gh1 = S.hl;
      if (C > 1) {
        for (int i = tid; i < kBins; i += kThreads) {
          const uint32_t v = S.hl[i];
          if (v) red_add_cluster(S.gh1 + i, 0, v);
        }
        cluster.sync();
        gh1 = cluster.map_shared_rank(S.gh1, 0);
      }
      find_digit<4>(gh1, k_rem, S.wsum, &S.found);
      prefix |= S.found.digit << 10;
      mask |= 0x7ffu << 10;
      k_rem -= S.found.above;
      done = (S.found.eq == k_rem);
    }
    // ---- digit 3 ----
    if (!done) {
      for (int i = tid; i < kBins / 2; i += kThreads) S.hl[i] = 0u;
      if (!ovf1) {
        for (uint32_t e0 = 0; e0 < n1; e0 += kThreads) {
          const uint32_t e = e0 + tid;
          const uint32_t key = e < n1 ? S.cand[e] : 0u;
          list_append(S.cand2, &S.ctl.cnt2, kCand2Cap, key, e < n1 && (key & mask) == prefix);
        }
      } else {
        for (int t = 0; t < ntiles; ++t) {
          uint32_t k[kPerThread];
          load_tile(gk, len, t, k);
          const int li = t * kTile + tid * kPerThread;
#pragma unroll
          for (int e = 0; e < kPerThread; ++e)
            list_append(S.cand2, &S.ctl.cnt2, kCand2Cap, k[e], li + e < len && (k[e] & mask) == prefix);
        }
      }
      __syncthreads();
      const uint32_t n2 = S.ctl.cnt2;
      if (n2 <= (uint32_t)kCand2Cap) {
        for (uint32_t e0 = 0; e0 < n2; e0 += kThreads) {
          const uint32_t e = e0 + tid;
          const uint32_t key = e < n2 ? S.cand2[e] : 0u;
          hist_add(S.hl, key & 0x3ffu, e < n2);
        }
      } else {
        for (int t = 0; t < ntiles; ++t) {
          uint32_t k[kPerThread];
          load_tile(gk, len, t, k);
          const int li = t * kTile + tid * kPerThread;
#pragma unroll
          for (int e = 0; e < kPerThread; ++e)
            hist_add(S.hl, k[e] & 0x3ffu, li + e < len && (k[e] & mask) == prefix);
        }
      }
      __syncthreads();
      const uint32_t* gh2 = S.hl;
      if (C > 1) {
        for (int i = tid; i < kBins / 2; i += kThreads) {
          const uint32_t v = S.hl[i];
          if (v) red_add_cluster(S.gh2 + i, 0, v);
        }
        cluster.sync();
        gh2 = cluster.map_shared_rank(S.gh2, 0);
      }
      find_digit<2>(gh2, k_rem, S.wsum, &S.found);
      prefix |= S.found.digit;
      mask = 0xffffffffu;
      k_rem -= S.found.above;
    }
    const uint32_t need = k_rem;  // how many of the threshold-key positions to take

    // ---- CTA totals: above the threshold, equal to it ----
    uint32_t my_gt = gt0, my_eq = 0u;
    if (done && mask == (0x7ffu << 21)) {
      my_eq = eq0;  // the first digit settled the threshold: its whole bin is selected
    } else if (!ovf1) {
      // keys above digit 1 are all above the threshold; the rest is among the candidates
      for (uint32_t e = tid; e < n1; e += kThreads) {
        const uint32_t m = S.cand[e] & mask;
        my_gt += (m > prefix) ? 1u : 0u;
        my_eq += (m == prefix) ? 1u : 0u;
      }
    } else {
      my_gt = 0u;
      for (int t = 0; t < ntiles; ++t) {
        uint32_t k[kPerThread];
        load_tile(gk, len, t, k);
        const int li = t * kTile + tid * kPerThread;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          const uint32_t m = k[e] & mask;
          const bool valid = li + e < len;
          my_gt += (valid && m > prefix) ? 1u : 0u;
          my_eq += (valid && m == prefix) ? 1u : 0u;
        }
      }
    }
    const uint32_t cta_gt = block_sum(my_gt, S.wsum);
    const uint32_t cta_eq = block_sum(my_eq, S.wsum);
    if (tid == 0) {
      S.ctl.cta_gt = cta_gt;
      S.ctl.cta_eq = cta_eq;
    }
    uint32_t gt_base = 0u, eq_base = 0u;
    if (C > 1) {
      cluster.sync();
      if (tid < 32) {
        uint32_t gb = 0u, eb = 0u;
        if (tid < rank) {
          const Ctl* rc = cluster.map_shared_rank(&S.ctl, tid);
          gb = rc->cta_gt;
          eb = rc->cta_eq;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          gb += __shfl_xor_sync(0xffffffffu, gb, o);
          eb += __shfl_xor_sync(0xffffffffu, eb, o);
        }
        if (tid == 0) {
          S.ctl.gt_before = gb;
          S.ctl.eq_before = eb;
        }
      }
      __syncthreads();
      gt_base = S.ctl.gt_before;
      eq_base = S.ctl.eq_before;
    }

    // ---- pass 2 over the chunk: ordered compaction, one block scan per tile ----
    {
      uint32_t cur[kPerThread];
#pragma unroll
      for (int e = 0; e < kPerThread; ++e) cur[e] = 0u;
      if (ntiles > 0) load_tile(gk, len, 0, cur);
      for (int t = 0; t < ntiles; ++t) {
        uint32_t nxt[kPerThread];
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) nxt[e] = 0u;
        if (t + 1 < ntiles) load_tile(gk, len, t + 1, nxt);
        const int li = t * kTile + tid * kPerThread;
        uint32_t tg = 0u, te = 0u;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          const uint32_t m = cur[e] & mask;
          const bool valid = li + e < len;
          tg += (valid && m > prefix) ? 1u : 0u;
          te += (valid && m == prefix) ? 1u : 0u;
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan((tg << 16) | te, S.wsum, &tot);
        uint32_t gc = gt_base + (ex >> 16);
        uint32_t ec = eq_base + (ex & 0xffffu);
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          const uint32_t m = cur[e] & mask;
          if (li + e < len) {
            const int pos = c0 + li + e;
            if (m > prefix) {
              idx[gc + min(ec, need)] = pos;
              ++gc;
            } else if (m == prefix) {
              if (ec < need) idx[gc + ec] = pos;
              ++ec;
            }
          }
        }
        gt_base += tot >> 16;
        eq_base += tot & 0xffffu;
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) cur[e] = nxt[e];
      }
    }
    for (int j = k_eff + rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = -1;
    if (C > 1) cluster.sync();  // peers may still read this CTA's shared memory
  }
}

}  // namespace

bool plan_select(SelectParams& p, int num_sms) {
  const int heads = p.B * p.Hkv;
  // Double the CTAs per head while the grid still fits one wave of two CTAs per SM and each
  // CTA keeps at least one tile of keys.
  int C = 1;
  while (C < kMaxCluster && (long)heads * C * 2 <= 2L * num_sms && (p.cap + 2 * C - 1) / (2 * C) >= kTile) C *= 2;
  p.cluster = C;
  p.chunk = (((p.cap + C - 1) / C) + 15) & ~15;
  p.cand_cap = kCandCap;
  p.off_hist = 0;
  p.off_ctl = 0;
  p.smem_bytes = (int)sizeof(SelSmem);
  return true;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  auto kern = select_topk_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
  if (e != cudaSuccess) return e;
  if (p.cluster > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.cluster, (unsigned)(p.B * p.Hkv), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace sas
