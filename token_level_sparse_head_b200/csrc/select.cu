// Per-KV-head top-k selection over the score keys (sm_100a).
//
// JSSA page, section JSSA 的整体结构 / Figure 1: every KV head keeps the positions of its k
// largest projected scores, and its G query heads share them; section 局限与需要留意的地方:
// no sink or recent window is forced.  The score kernel has left each (b, h)'s order-preserving
// uint32 keys in the workspace (on chip in L2) together with a histogram of their top 11 bits.
//
// One thread-block cluster per (b, h); each CTA copies a contiguous chunk of the keys into
// shared memory.  The k-th largest key is found digit by digit (11, 11, 10 bits):
//   digit 1 straight from the global histogram (every CTA computes the same answer);
//   digits 2 and 3 from histograms of the surviving candidates only, which each CTA adds into
//   rank 0's shared memory with fire-and-forget cluster reductions, one cluster barrier each.
// A digit whose bin holds exactly the remaining count ends the search.  Then an ordered
// compaction: positions with a larger key are selected, and of those equal to the threshold key
// the lowest positions fill the remainder (exact ties -> lower position).  A cluster-wide
// exclusive count gives every position its output slot, so the index list comes out ascending
// with no sort.
#include <cooperative_groups.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace cg = cooperative_groups;

namespace sas {
namespace {

constexpr int kThreads = 256;
constexpr int kBins = 2048;      // 11-bit digits
constexpr int kCand2 = 2048;     // survivors of the second digit kept on chip

struct Ctl {
  uint32_t cnt1, cnt2, pad0, pad1;
  uint32_t cta_gt, cta_eq, gt_before, eq_before;
};

// Exclusive prefix sum over the 256 threads of the block; *total receives the block sum.
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
  for (int w = 0; w < kThreads / 32; ++w) {
    const uint32_t s = wsum[w];
    off += (w < warp) ? s : 0u;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return off + x - v;
}

// Warp-aggregated shared-memory histogram increment (many lanes share few bins).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  const int lane = threadIdx.x & 31;
  if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Digit holding the k_rem-th largest key, from a histogram of `nb` bins (2048 or 1024) that may
// live in another CTA's shared memory.  Every CTA of a cluster runs this on the same histogram
// and gets the same answer.  Thread t covers digits [nb - (t+1)*per, nb - t*per).
struct Found {
  uint32_t digit, above, eq, pad;
};

template <int PER>
__device__ __forceinline__ void find_digit(const uint32_t* H, uint32_t k_rem, uint32_t* wsum, Found* out) {
  const int tid = threadIdx.x;
  const int lo = PER * kThreads - (tid + 1) * PER;  // first digit of my range (nb = PER * 256)
  uint32_t c[PER];
  if constexpr (PER == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(H + lo);
    const uint4 b = *reinterpret_cast<const uint4*>(H + lo + 4);
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(H + lo);
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
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

// Fire-and-forget add into the same shared-memory word of cluster CTA `rank`.
__device__ __forceinline__ void red_add_cluster(const uint32_t* local, uint32_t rank, uint32_t v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(ra), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kThreads) select_topk_kernel(const SelectParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int C = (int)cluster.num_blocks();
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;

  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  uint32_t* hl = reinterpret_cast<uint32_t*>(smem + p.off_hist);  // this CTA's histogram
  uint32_t* gh1 = hl + kBins;                                       // rank 0: cluster histogram, digit 2
  uint32_t* gh2 = gh1 + kBins;                                      // rank 0: cluster histogram, digit 3
  uint32_t* cand2 = gh2 + kBins / 2;
  uint32_t* cand = cand2 + kCand2;
  const uint32_t cap1 = (uint32_t)p.cand_cap;
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + p.off_ctl);
  Found* found = reinterpret_cast<Found*>(ctl + 1);
  uint32_t* wsum = reinterpret_cast<uint32_t*>(found + 1);

  // per-sequence values (range errors were recorded by the score kernel)
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) n = 0;
  const int kb = min(p.kvec[b], p.k_max);
  const int k_eff = max(0, min(kb, n));
  int32_t* idx = p.idx_out + (size_t)bh * p.k_max;

  // Nothing to rank: empty selection, or every position selected.  Uniform per cluster.
  if (k_eff == 0 || k_eff == n) {
    for (int j = rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = (j < k_eff) ? j : -1;
    return;
  }

  // ---- this CTA's positions [c0, c1) ----
  const int chunk_b = ((n + C - 1) / C + 511) & ~511;  // multiple of 512 -> even run
  const int run = chunk_b / kThreads;                  // positions per thread
  const int c0 = min(rank * chunk_b, n);
  const int c1 = min(c0 + chunk_b, n);
  const int len = c1 - c0;
  const int my0 = tid * run;

  // ---- keys of the chunk into shared memory (padded: one spare word per run) ----
  const uint32_t* gk = p.keys + (size_t)bh * p.cap + c0;
  for (int v = tid; v * 4 < len; v += kThreads) {
    const int li = v * 4;
    if (li + 4 <= len) {
      const uint4 w = *reinterpret_cast<const uint4*>(gk + li);
      keys[li + li / run] = w.x;
      keys[li + 1 + (li + 1) / run] = w.y;
      keys[li + 2 + (li + 2) / run] = w.z;
      keys[li + 3 + (li + 3) / run] = w.w;
    } else {
      for (int e = li; e < len; ++e) keys[e + e / run] = gk[e];
    }
  }
  for (int i = tid; i < kBins + kBins + kBins / 2; i += kThreads) hl[i] = 0u;  // hl, gh1, gh2
  if (tid == 0) {
    ctl->cnt1 = 0u;
    ctl->cnt2 = 0u;
  }

  // ---- digit 1 from the global histogram (identical in every CTA of the cluster) ----
  const uint32_t* ghist = p.hist + (size_t)bh * kBins;
  uint32_t k_rem = (uint32_t)k_eff;
  find_digit<8>(ghist, k_rem, wsum, found);  // ends with __syncthreads: keys, zeros visible
  uint32_t prefix = found->digit << 21;
  uint32_t mask = 0x7ffu << 21;
  k_rem -= found->above;
  bool done = (found->eq == k_rem);
  // Every CTA has read the global histogram and zeroed its cluster histograms: after this
  // barrier, rank 0 clears the global histogram for the next call and the adds can start.
  cluster.sync();
  if (rank == 0)
    for (int i = tid; i < kBins; i += kThreads) const_cast<uint32_t*>(ghist)[i] = 0u;

  bool ovf1 = false;
  if (!done) {
    // candidates: the keys in the threshold bin of digit 1
    for (int i = 0; i < run; ++i) {
      const int li = my0 + i;
      const uint32_t key = li < len ? keys[li + tid] : 0u;
      list_append(cand, &ctl->cnt1, cap1, key, li < len && (key & mask) == prefix);
    }
    __syncthreads();
    const uint32_t n1 = ctl->cnt1;
    ovf1 = n1 > cap1;
    if (!ovf1) {
      for (uint32_t e0 = 0; e0 < n1; e0 += kThreads) {
        const uint32_t e = e0 + tid;
        const uint32_t key = e < n1 ? cand[e] : 0u;
        hist_add(hl, (key >> 10) & 0x7ffu, e < n1);
      }
    } else {
      for (int i = 0; i < run; ++i) {
        const int li = my0 + i;
        const uint32_t key = li < len ? keys[li + tid] : 0u;
        hist_add(hl, (key >> 10) & 0x7ffu, li < len && (key & mask) == prefix);
      }
    }
    __syncthreads();
    for (int i = tid; i < kBins; i += kThreads) {
      const uint32_t v = hl[i];
      if (v) red_add_cluster(gh1 + i, 0, v);
    }
    cluster.sync();
    find_digit<8>(cluster.map_shared_rank(gh1, 0), k_rem, wsum, found);
    prefix |= found->digit << 10;
    mask |= 0x7ffu << 10;
    k_rem -= found->above;
    done = (found->eq == k_rem);
  }
  if (!done) {
    // survivors of digit 2
    for (int i = tid; i < kBins / 2; i += kThreads) hl[i] = 0u;
    if (!ovf1) {
      const uint32_t n1 = ctl->cnt1;
      for (uint32_t e0 = 0; e0 < n1; e0 += kThreads) {
        const uint32_t e = e0 + tid;
        const uint32_t key = e < n1 ? cand[e] : 0u;
        list_append(cand2, &ctl->cnt2, kCand2, key, e < n1 && (key & mask) == prefix);
      }
    } else {
      for (int i = 0; i < run; ++i) {
        const int li = my0 + i;
        const uint32_t key = li < len ? keys[li + tid] : 0u;
        list_append(cand2, &ctl->cnt2, kCand2, key, li < len && (key & mask) == prefix);
      }
    }
    __syncthreads();
    const uint32_t n2 = ctl->cnt2;
    if (n2 <= kCand2) {
      for (uint32_t e0 = 0; e0 < n2; e0 += kThreads) {
        const uint32_t e = e0 + tid;
        const uint32_t key = e < n2 ? cand2[e] : 0u;
        hist_add(hl, key & 0x3ffu, e < n2);
      }
    } else {
      for (int i = 0; i < run; ++i) {
        const int li = my0 + i;
        const uint32_t key = li < len ? keys[li + tid] : 0u;
        hist_add(hl, key & 0x3ffu, li < len && (key & mask) == prefix);
      }
    }
    __syncthreads();
    for (int i = tid; i < kBins / 2; i += kThreads) {
      const uint32_t v = hl[i];
      if (v) red_add_cluster(gh2 + i, 0, v);
    }
    cluster.sync();
    find_digit<4>(cluster.map_shared_rank(gh2, 0), k_rem, wsum, found);
    prefix |= found->digit;
    mask = 0xffffffffu;
    k_rem -= found->above;
  }

  // ---- ordered compaction ----
  const uint32_t need = k_rem;  // how many of the threshold-key positions to take
  uint32_t n_gt = 0u, n_eq = 0u;
  for (int i = 0; i < run; ++i) {
    const int li = my0 + i;
    if (li < len) {
      const uint32_t m = keys[li + tid] & mask;
      n_gt += (m > prefix);
      n_eq += (m == prefix);
    }
  }
  uint32_t tot;
  const uint32_t excl = block_excl_scan((n_gt << 16) | n_eq, wsum, &tot);
  if (tid == 0) {
    ctl->cta_gt = tot >> 16;
    ctl->cta_eq = tot & 0xffffu;
  }
  cluster.sync();
  if (tid < 32) {
    uint32_t gb = 0u, eb = 0u;
    if (tid < rank) {
      const Ctl* rc = cluster.map_shared_rank(ctl, tid);
      gb = rc->cta_gt;
      eb = rc->cta_eq;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      gb += __shfl_xor_sync(0xffffffffu, gb, o);
      eb += __shfl_xor_sync(0xffffffffu, eb, o);
    }
    if (tid == 0) {
      ctl->gt_before = gb;
      ctl->eq_before = eb;
    }
  }
  __syncthreads();
  uint32_t gt_c = ctl->gt_before + (excl >> 16);
  uint32_t eq_c = ctl->eq_before + (excl & 0xffffu);
  for (int i = 0; i < run; ++i) {
    const int li = my0 + i;
    if (li < len) {
      const uint32_t m = keys[li + tid] & mask;
      const int pos = c0 + li;
      if (m > prefix) {
        idx[gt_c + min(eq_c, need)] = pos;
        ++gt_c;
      } else if (m == prefix) {
        if (eq_c < need) idx[gt_c + eq_c] = pos;
        ++eq_c;
      }
    }
  }
  for (int j = k_eff + rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = -1;
  cluster.sync();  // peers may still read this CTA's shared memory
}

cudaError_t launch_sel(const SelectParams& p, cudaStream_t stream) {
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

}  // namespace

bool plan_select(SelectParams& p, int num_sms) {
  const int cap = p.cap;
  const int heads = p.B * p.Hkv;
  int C = 1;
  auto chunk_of = [&](int c) { return (((cap + c - 1) / c) + 511) & ~511; };
  while (C < kMaxCluster && chunk_of(C) > 8192) C *= 2;
  while (C < kMaxCluster && (long)heads * C < 2L * num_sms && (cap + 2 * C - 1) / (2 * C) >= 1024) C *= 2;
  const int chunk = chunk_of(C);
  if (chunk > kMaxChunk) return false;
  p.cluster = C;
  p.chunk = chunk;
  p.cand_cap = chunk / 4 > 1024 ? chunk / 4 : 1024;
  const int keys_bytes = ((chunk + kThreads) * 4 + 127) & ~127;
  p.off_hist = keys_bytes;
  const int hist_bytes = (kBins + kBins + kBins / 2 + kCand2 + p.cand_cap) * 4;
  p.off_ctl = p.off_hist + ((hist_bytes + 15) & ~15);
  p.smem_bytes = p.off_ctl + (int)sizeof(Ctl) + (int)sizeof(Found) + (kThreads / 32) * 4;
  return p.smem_bytes <= 227 * 1024;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) { return launch_sel(p, stream); }

}  // namespace sas
