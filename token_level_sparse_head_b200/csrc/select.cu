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
constexpr int kStep = 16;            // keys per thread per step (four 16-byte loads)
constexpr int kMaxRun = 256;         // keys per thread at most (the plan sizes clusters for it)
constexpr int kWords = kMaxRun / 32; // per-thread position bitmask words
constexpr int kOwnCand = 16;         // candidate keys kept on chip per thread

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
  uint32_t cand[kOwnCand][kThreads];  // per-thread candidate keys, in position order
  uint32_t wsum[kWarps];
  unsigned long long wsum64[kWarps];
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

// Exclusive prefix sum of 64-bit values over the block; *total receives the block sum.
__device__ __forceinline__ unsigned long long block_excl_scan64(unsigned long long v, unsigned long long* wsum,
                                                                unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  unsigned long long off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned long long s = wsum[w];
    off += (w < warp) ? s : 0ull;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return off + x - v;
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

// Step i of this thread's contiguous run: keys [base + 16 i, +16) of the chunk; positions past
// the run or the chunk read as 0 (and are masked by the callers).  Cached loads: the four
// 16-byte loads of a step share 32-byte sectors.
__device__ __forceinline__ void load_step(const uint32_t* gk, int base, int end, int i, uint32_t (&k)[kStep]) {
  const int li = base + i * kStep;
  if (li + kStep <= end) {
#pragma unroll
    for (int v = 0; v < kStep / 4; ++v) {
      const uint4 a = *reinterpret_cast<const uint4*>(gk + li + 4 * v);
      k[4 * v + 0] = a.x; k[4 * v + 1] = a.y; k[4 * v + 2] = a.z; k[4 * v + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kStep; ++e) k[e] = (li + e < end) ? gk[li + e] : 0u;
  }
}

// Bit e of the result is set where positions base + e (e < 16) lie before `end`.
__device__ __forceinline__ uint32_t valid_bits(int base, int end) {
  const int n = end - base;
  return n >= kStep ? 0xffffu : (n > 0 ? ((1u << n) - 1u) : 0u);
}

// Bitmasks of the keys k[e] with (k & mask) above / equal to `prefix`.
__device__ __forceinline__ void step_masks(const uint32_t (&k)[kStep], uint32_t mask, uint32_t prefix,
                                           uint32_t& above, uint32_t& equal) {
  above = 0u;
  equal = 0u;
#pragma unroll
  for (int e = 0; e < kStep; ++e) {
    const uint32_t m = k[e] & mask;
    above |= (m > prefix ? 1u : 0u) << e;
    equal |= (m == prefix ? 1u : 0u) << e;
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

  // this CTA's positions [c0, c1); each thread owns a contiguous run of K of them
  const int chunk_b = (((n + C - 1) / C) + 15) & ~15;
  const int c0 = min(rank * chunk_b, n);
  const int c1 = min(c0 + chunk_b, n);
  const int len = c1 - c0;
  const uint32_t* gk = p.keys + (size_t)bh * p.cap + c0;
  const int K = ((len + kThreads - 1) / kThreads + kStep - 1) / kStep * kStep;
  const int my0 = min(tid * K, len);
  const int my1 = min(my0 + K, len);
  const int nsteps = (my1 - my0 + kStep - 1) / kStep;
  const int lane = tid & 31, warp = tid >> 5;

  if (trivial) {
    for (int j = rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = (j < k_eff) ? j : -1;
  } else {
    // Bring the whole chunk of keys towards the SM early: the L2 fetches them from DRAM in
    // large runs while the digit search below runs.
    if (warp == 0) {
      const int bytes = ((len * 4) + 15) & ~15;
      for (int o = lane * 8192; o < bytes; o += 32 * 8192)
        bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(gk) + o, (uint32_t)min(8192, bytes - o));
    }
    for (int i = tid; i < kBins + kBins + kBins / 2; i += kThreads) S.hl[i] = 0u;  // hl, gh1, gh2
    // ---- digit 1 from the global histogram ----
    const uint32_t* ghist = p.hist + (size_t)bh * kBins;
    uint32_t k_rem = (uint32_t)k_eff;
    find_digit<4>(ghist, k_rem, S.wsum, &S.found);
    const uint32_t d0 = S.found.digit;
    uint32_t prefix = d0 << 21;
    uint32_t mask = 0x7ffu << 21;
    k_rem -= S.found.above;
    bool done = (S.found.eq == k_rem);
    const bool done1 = done;

    // ---- the one read of my run: bitmasks of the keys above digit 1 (gtm) and equal to it
    // (cm); the equal ones (candidates) are also kept, in position order, in my slot ----
    uint32_t gtm[kWords], cm[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) {
      gtm[w] = 0u;
      cm[w] = 0u;
    }
    uint32_t nc = 0u;  // my candidates (beyond kOwnCand: keys re-read when needed)
    for (int i = 0; i < nsteps; ++i) {
      uint32_t k[kStep];
      load_step(gk, my0, my1, i, k);
      uint32_t sg, sc;
      step_masks(k, 0x7ffu << 21, d0 << 21, sg, sc);
      const uint32_t vb = valid_bits(my0 + i * kStep, my1);
      sg &= vb;
      sc &= vb;
      const int sh = (i & 1) * kStep;
#pragma unroll
      for (int w = 0; w < kWords; ++w) {
        if (w == (i >> 1)) {
          gtm[w] |= sg << sh;
          cm[w] |= sc << sh;
        }
      }
      if (sc != 0u && !done) {
#pragma unroll
        for (int e = 0; e < kStep; ++e) {
          if ((sc >> e) & 1u) {
            if (nc < (uint32_t)kOwnCand) S.cand[nc][tid] = k[e];
            ++nc;
          }
        }
      }
    }
    const bool own_ovf = nc > (uint32_t)kOwnCand;
    const uint32_t nown = min(nc, (uint32_t)kOwnCand);
    __syncthreads();
    // Every CTA has read the global histogram and zeroed its cluster histograms: after this
    // barrier rank 0 clears the global histogram for the next call, and the adds may start.
    if (C > 1) cluster.sync();
    if (rank == 0)
      for (int i = tid; i < kBins; i += kThreads) const_cast<uint32_t*>(ghist)[i] = 0u;

    // Histogram of digit `shift` (11 bits at 10, or 10 bits at 0) of my candidates that match
    // the current prefix, into hl: from my slot, or by re-reading my run when it overflowed.
    auto cand_hist = [&](int shift, uint32_t dmask) {
#pragma unroll
      for (int j = 0; j < kOwnCand; ++j) {
        const uint32_t key = S.cand[j][tid];
        const bool act = !own_ovf && (uint32_t)j < nown && (key & mask) == prefix;
        hist_add(S.hl, (key >> shift) & dmask, act);
      }
      if (own_ovf) {
        for (int i = 0; i < nsteps; ++i) {
          uint32_t k[kStep];
          load_step(gk, my0, my1, i, k);
          const int li = my0 + i * kStep;
#pragma unroll
          for (int e = 0; e < kStep; ++e)
            if (li + e < my1 && (k[e] & mask) == prefix) atomicAdd(&S.hl[(k[e] >> shift) & dmask], 1u);
        }
      }
    };

    // ---- digit 2 ----
    if (!done) {
      cand_hist(10, 0x7ffu);
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
      __syncthreads();
      cand_hist(0, 0x3ffu);
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

    // The key of my j-th candidate (position order), from my slot or from memory.
    auto own_key = [&](uint32_t j, int pos_in_chunk) -> uint32_t {
      return own_ovf ? gk[pos_in_chunk] : S.cand[j][tid];
    };

    // ---- my counts above / equal to the threshold ----
    uint32_t my_gt = 0u, my_eq = 0u;
#pragma unroll
    for (int w = 0; w < kWords; ++w) {
      my_gt += (uint32_t)__popc(gtm[w]);
      my_eq += (uint32_t)__popc(cm[w]);
    }
    if (!done1) {
      // the candidates split by their full keys
      uint32_t cgt = 0u, ceq = 0u, j = 0u;
#pragma unroll
      for (int w = 0; w < kWords; ++w) {
        uint32_t bits = cm[w];
        while (bits) {
          const int bpos = __ffs(bits) - 1;
          bits &= bits - 1u;
          const uint32_t m = own_key(j, my0 + w * 32 + bpos) & mask;
          ++j;
          cgt += (m > prefix) ? 1u : 0u;
          ceq += (m == prefix) ? 1u : 0u;
        }
      }
      my_gt += cgt;
      my_eq = ceq;
    }
    unsigned long long tot;
    const unsigned long long ex =
        block_excl_scan64(((unsigned long long)my_gt << 32) | my_eq, S.wsum64, &tot);
    if (tid == 0) {
      S.ctl.cta_gt = (uint32_t)(tot >> 32);
      S.ctl.cta_eq = (uint32_t)tot;
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

    // ---- write my selected positions in order (no further reads unless my slot overflowed) ----
    {
      uint32_t gc = gt_base + (uint32_t)(ex >> 32);
      uint32_t ec = eq_base + (uint32_t)ex;
      uint32_t j = 0u;
#pragma unroll
      for (int w = 0; w < kWords; ++w) {
        uint32_t bits = gtm[w] | cm[w];
        while (bits) {
          const int bpos = __ffs(bits) - 1;
          bits &= bits - 1u;
          const int pic = my0 + w * 32 + bpos;  // position in the chunk
          bool above, equal;
          if ((gtm[w] >> bpos) & 1u) {
            above = true;
            equal = false;
          } else if (done1) {
            above = false;
            equal = true;
          } else {
            const uint32_t m = own_key(j, pic) & mask;
            above = m > prefix;
            equal = m == prefix;
          }
          if (!((gtm[w] >> bpos) & 1u)) ++j;
          if (above) {
            idx[gc + min(ec, need)] = c0 + pic;
            ++gc;
          } else if (equal) {
            if (ec < need) idx[gc + ec] = c0 + pic;
            ++ec;
          }
        }
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
  while (C < kMaxCluster && (p.cap + C - 1) / C > kThreads * kMaxRun) C *= 2;
  while (C < kMaxCluster && (long)heads * C * 2 <= 2L * num_sms && (p.cap + 2 * C - 1) / (2 * C) >= kThreads * kStep) C *= 2;
  if ((p.cap + C - 1) / C > kThreads * kMaxRun) return false;
  p.cluster = C;
  p.chunk = (((p.cap + C - 1) / C) + 15) & ~15;
  p.cand_cap = kThreads * kOwnCand;
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
