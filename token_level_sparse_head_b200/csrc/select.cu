// Per-KV-head top-k selection over the score keys (sm_100a).
//
// JSSA page, section JSSA 的整体结构 / Figure 1: every KV head keeps the positions of its k
// largest projected scores, and its G query heads share them; section 局限与需要留意的地方:
// no sink or recent window is forced.  The score kernel has left each (b, h)'s order-preserving
// uint32 keys in the workspace (in L2) with a histogram of their first 13 bits.
//
// A cluster of C CTAs serves one (b, h) (C = 1 when there are enough heads to fill the GPU);
// each CTA owns a contiguous chunk of positions.  The k-th largest key T is found as three radix
// digits (13, 10 and 9 bits); ties on T go to the lower positions.
//   1. The global histogram gives digit 1.  Each CTA streams its chunk of keys once: every warp
//      takes tiles of 512 keys in turn through a shared-memory ring of its own (bulk copies;
//      each lane turns 16 keys into 16 bits of a bitmap word), setting a position bitmap of the
//      keys whose digit 1 is larger (they are selected) and appending the keys whose digit 1
//      equals it (the candidates, a few percent of the positions) to a list.
//   2. The candidate lists are gathered into CTA 0 of the cluster through distributed shared
//      memory; CTA 0 finds digits 2 and 3 among them, resolves the ties, marks the chosen
//      candidates in the owners' bitmaps and hands every CTA its first output slot.
//   3. Each CTA writes the set bits of its bitmap, in order, as ascending positions.
// When the candidates do not fit the list, or many keys tie on T, every CTA re-reads its keys
// instead (a slower path with the same result).
#include <cooperative_groups.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace cg = cooperative_groups;

namespace sas {
namespace {

constexpr int kBins2 = 1 << kDigit2Bits;      // 1024
constexpr int kBins3 = 1 << kDigit3Bits;      // 512
constexpr int kChunkMax = 131072;             // positions per CTA at most
constexpr int kMaxWords = kChunkMax / 32;     // bitmap words per CTA
constexpr int kCap = 4096;                    // candidate list entries (CTA 0: the whole head's)
constexpr int kMaxTies = 256;                 // ties on T resolved by CTA 0; more take the slow path
constexpr uint32_t kFast = 1u, kSlow = 2u;

struct Found {
  uint32_t digit, above, eq, pad;
};

struct Ctl {
  uint32_t ccount;   // candidates appended to this CTA's list (CTA 0: gathered from the cluster)
  uint32_t above;    // keys of this CTA above digit 1
  uint32_t flag;     // written by CTA 0: kFast (base valid) or kSlow
  uint32_t base;     // written by CTA 0: first output slot of this CTA
  uint32_t ntie;
  int32_t tie_cut;   // ties at positions <= tie_cut are taken
  uint32_t pad[2];
  uint32_t above_of[kMaxCluster];  // CTA 0: per-CTA counts
  uint32_t sel_of[kMaxCluster];
  uint32_t tie_of[kMaxCluster];
};

// Block shape: THREADS threads per CTA.  1024 threads serve a head per CTA (B=16); clusters of
// several CTAs per head (small batches) use 512, which spend less time in block-wide barriers.
// Each warp streams its own tiles of 512 keys (2 KB) through a ring of its own, kSlots deep, so
// 128 KB of keys are in flight per CTA either way.
template <int THREADS>
struct Cfg {
  static constexpr int kThreads = THREADS;
  static constexpr int kWarps = THREADS / 32;
  static constexpr int kTileKeys = 512;            // keys per tile: 16 per lane
  static constexpr int kSlots = 2 * 1024 / THREADS;
};

template <int THREADS>
struct SelSmem {
  static constexpr int kSlots = Cfg<THREADS>::kSlots;
  static constexpr int kWarps = Cfg<THREADS>::kWarps;
  uint32_t ring[kWarps][kSlots][Cfg<THREADS>::kTileKeys];
  uint32_t bm[kMaxWords];     // selected positions of the chunk
  uint32_t ckey[kCap];        // candidate keys (slow path: tie bits per bitmap word)
  int32_t cpos[kCap];         // candidate positions in the head
  uint32_t hloc[kBins2];
  uint32_t hacc2[kBins2];     // CTA 0, slow path: cluster histogram of digit 2
  uint32_t hacc3[kBins3];     // CTA 0: histogram of digit 3
  int32_t tpos[kMaxTies];
  uint64_t full[kWarps][kSlots];
  uint32_t wsum[kWarps];
  Ctl ctl;
  Found found;
};

// Exclusive prefix sum over the block; *total receives the block sum.  Warp sums meet in shared
// memory and every warp scans them with shuffles (at most 32 of them).
template <int THREADS>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  constexpr int kWarps = THREADS / 32;
  static_assert(kWarps <= 32, "one warp sum per lane");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  const uint32_t ws = lane < kWarps ? wsum[lane] : 0u;
  uint32_t wi = ws;
#pragma unroll
  for (int o = 1; o < kWarps; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
    if (lane >= o) wi += y;
  }
  const uint32_t off = __shfl_sync(0xffffffffu, wi - ws, warp);
  *total = __shfl_sync(0xffffffffu, wi, kWarps - 1);
  __syncthreads();  // wsum may be written again by the next scan
  return off + x - v;
}

// Digit holding the k_rem-th largest key, from a histogram of NB bins read through a generic
// pointer (this CTA's shared memory, CTA 0's through the cluster, or global memory).  Thread t
// covers digits [NB - (t+1)*PER, NB - t*PER), highest first (threads past NB / PER hold none).
// Writes *out (digit, count above it, count in it); out is left unchanged if the histogram
// holds fewer keys.
template <int NB, int THREADS>
__device__ __forceinline__ void find_digit(const uint32_t* H, uint32_t k_rem, uint32_t* wsum, Found* out) {
  constexpr int kThreads = THREADS;
  constexpr int PER = NB >= kThreads ? NB / kThreads : 1;
  constexpr int ACT = NB / PER;
  const int lo = NB - ((int)threadIdx.x + 1) * PER;
  uint32_t c[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) c[j] = 0u;
  if ((int)threadIdx.x < ACT) {
    if constexpr (PER % 4 == 0) {
#pragma unroll
      for (int q = 0; q < PER / 4; ++q) {
        const uint4 a = reinterpret_cast<const uint4*>(H + lo)[q];
        c[4 * q] = a.x; c[4 * q + 1] = a.y; c[4 * q + 2] = a.z; c[4 * q + 3] = a.w;
      }
    } else if constexpr (PER == 2) {
      const uint2 a = *reinterpret_cast<const uint2*>(H + lo);
      c[0] = a.x; c[1] = a.y;
    } else {
      c[0] = H[lo];
    }
  }
  uint32_t tsum = 0u;
#pragma unroll
  for (int j = 0; j < PER; ++j) tsum += c[j];
  uint32_t tot;
  const uint32_t above = block_excl_scan<THREADS>(tsum, wsum, &tot);
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

// ---- distributed shared memory (cluster) primitives ----
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  return ra;
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t dsmem_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t dsmem_atomic_add(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void dsmem_red_add(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void dsmem_red_or(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.or.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Split cluster barrier: arrive (release) now, wait (acquire) later.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS, 1) select_topk_kernel(const SelectParams p) {
  constexpr int kThreads = Cfg<THREADS>::kThreads;
  constexpr int kWarps = Cfg<THREADS>::kWarps;
  constexpr int kTileKeys = Cfg<THREADS>::kTileKeys;
  constexpr int kSlots = Cfg<THREADS>::kSlots;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelSmem<THREADS>& S = *reinterpret_cast<SelSmem<THREADS>*>(smem_raw);
  const uint32_t rank = cg::this_cluster().block_rank();
  const int C = (int)cg::this_cluster().num_blocks();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;

  // per-sequence values (range errors were recorded by the score kernel)
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) n = 0;
  const SeqSelection sel = seq_selection(min(p.kvec[b], p.k_max), n);
  const int k_eff = sel.k_eff;
  int32_t* idx = p.idx_out + (size_t)bh * p.k_max;

  // this CTA's positions [c0, c1); chunks are whole bitmap words
  const int chunk = (((n + C - 1) / C) + 31) & ~31;
  const int c0 = min((int)rank * chunk, n);
  const int c1 = min(c0 + chunk, n);
  const int len = c1 - c0;
  const uint32_t* gk = p.keys + (size_t)bh * p.cap + c0;
  const int nwords = (len + 31) >> 5;
  const int wpt = (nwords + kThreads - 1) / kThreads;  // bitmap words per thread (<= 8)
  const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);

  if (!sel.ranked) {
    // Nothing to rank (uniform over the cluster): the first k_eff positions, or none.
    pdl_wait();
    pdl_trigger();
    for (int j = (int)rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = (j < k_eff) ? j : -1;
    return;
  }

  // ---------------------------------------------------------------- set-up
  // warp w streams tiles w, w + kWarps, ... of the chunk
  const int ntiles = (len + kTileKeys - 1) / kTileKeys;
  const int my_tiles = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;
  if (tid == 0) {
    for (int w = 0; w < kWarps; ++w)
      for (int s = 0; s < kSlots; ++s) mbar_init(&S.full[w][s], 1);
    fence_barrier_init();
  }
  for (int i = tid; i < kMaxWords; i += kThreads) S.bm[i] = 0u;
  for (int i = tid; i < kBins2; i += kThreads) {
    S.hloc[i] = 0u;
    S.hacc2[i] = 0u;
  }
  for (int i = tid; i < kBins3; i += kThreads) S.hacc3[i] = 0u;
  if (tid == 0) {
    Ctl z = {};
    z.tie_cut = 0x7fffffff;
    S.ctl = z;
    Found f = {};
    S.found = f;
  }
  __syncthreads();
  // The keys and histograms of the score pass are read only from here on.
  pdl_wait();
  pdl_trigger();

  // The warp's j-th tile (tile warp + j * kWarps of the chunk) into its slot j % kSlots, as whole
  // 16-byte units (the key rows have a multiple of 4 entries, so the rounding stays inside this
  // (b, h)'s row).  Issued by lane 0.
  auto issue = [&](int j) {
    const int t = warp + j * kWarps;
    const int slot = j % kSlots;
    const int keys = min(kTileKeys, len - t * kTileKeys);
    const uint32_t bytes = (uint32_t)((keys + 3) & ~3) * 4u;
    mbar_arrive_expect_tx(&S.full[warp][slot], bytes);
    bulk_g2s(S.ring[warp][slot], gk + (size_t)t * kTileKeys, bytes, &S.full[warp][slot]);
  };
  if (lane == 0)
    for (int j = 0; j < min(kSlots, my_tiles); ++j) issue(j);

  // ---- digit 1 from the global histogram ----
  const uint32_t* ghist = p.hist + (size_t)bh * kHistBins;
  find_digit<kHistBins, kThreads>(ghist, (uint32_t)k_eff, S.wsum, &S.found);
  const uint32_t d1 = S.found.digit;
  const uint32_t above1 = S.found.above;  // keys of the head with a larger digit 1
  const uint32_t eq1 = S.found.eq;        // keys of the head with this digit 1: the candidates
  const bool fast = eq1 <= (uint32_t)kCap;
  // One CTA per head: every thread has read the histogram (find_digit ends with a barrier), so
  // it is cleared for the next call now, under the streaming pass; in a cluster, CTA 0 clears it
  // once every CTA has passed the arrive below.
  if (C == 1)
    for (int i = tid; i < kHistBins / 4; i += kThreads)
      reinterpret_cast<uint4*>(const_cast<uint32_t*>(ghist))[i] = make_uint4(0u, 0u, 0u, 0u);
  cluster_arrive();  // this CTA's set-up is done and it has read the global histogram

  bool waited_ok = true;
  if (fast) {
    // ------------------------------------------------------------ streaming pass
    uint32_t my_above = 0u;
    // keys of digit d1 are [lo, hi]; above: key > hi (never true when d1 is the top digit)
    const uint32_t lo = d1 << kHistShift, hi = lo | ((1u << kHistShift) - 1u);
    for (int j = 0; j < my_tiles; ++j) {
      const int slot = j % kSlots;
      if (!mbar_wait_bounded(&S.full[warp][slot], (uint32_t)(j / kSlots) & 1u)) waited_ok = false;
      // lane l takes keys 16l .. 16l+15 of the tile: four 16-byte reads, lane pairs rotating
      // their order so that each read of the warp covers all banks; 2 lanes make a bitmap word
      const int t = warp + j * kWarps;
      const uint32_t* row = S.ring[warp][slot] + 16 * lane;
      const int lp = t * kTileKeys + 16 * lane;  // chunk position of the lane's first key
      uint32_t ab = 0u, cb = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = (q + (lane >> 1)) & 3;
        const uint4 kv = reinterpret_cast<const uint4*>(row)[c];
        const uint32_t k4[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t a4 = 0u, c4 = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a4 |= (k4[e] > hi ? 1u : 0u) << e;
          c4 |= (k4[e] - lo <= hi - lo ? 1u : 0u) << e;
        }
        ab |= a4 << (4 * c);
        cb |= c4 << (4 * c);
      }
      if ((t + 1) * kTileKeys > len) {  // the last, partial tile: drop keys past the chunk
        const uint32_t vm = (1u << min(max(len - lp, 0), 16)) - 1u;
        ab &= vm;
        cb &= vm;
      }
      uint32_t word = ab << (16 * (lane & 1));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      if ((lane & 1) == 0) S.bm[lp >> 5] = word;
      my_above += (uint32_t)__popc(ab);
      if (cb) {
        uint32_t jj = atomicAdd(&S.ctl.ccount, (uint32_t)__popc(cb));
        while (cb) {
          const int e = __ffs(cb) - 1;
          cb &= cb - 1u;
          if (jj < (uint32_t)kCap) {
            S.ckey[jj] = row[e];
            S.cpos[jj] = c0 + lp + e;
          }
          ++jj;
        }
      }
      __syncwarp();  // every lane is done with the slot
      if (lane == 0 && j + kSlots < my_tiles) issue(j + kSlots);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) my_above += __shfl_xor_sync(0xffffffffu, my_above, o);
    if (lane == 0 && my_above) atomicAdd(&S.ctl.above, my_above);
    __syncthreads();
    cluster_wait();  // every CTA of the cluster is set up: CTA 0's list may now be appended to
    if (C > 1 && rank == 0)
      for (int i = tid; i < kHistBins / 4; i += kThreads)
        reinterpret_cast<uint4*>(const_cast<uint32_t*>(ghist))[i] = make_uint4(0u, 0u, 0u, 0u);

    // ------------------------------------------------------------ gather into CTA 0
    const uint32_t mine = min(S.ctl.ccount, (uint32_t)kCap);
    if (rank != 0) {
      if (tid == 0) {
        const uint32_t base = dsmem_atomic_add(dsmem_addr(&S.ctl.ccount, 0), mine);
        S.ctl.ntie = base;  // this CTA's first slot in CTA 0's list (ntie is free here)
        dsmem_st(dsmem_addr(&S.ctl.above_of[rank], 0), S.ctl.above);
      }
      __syncthreads();
      const uint32_t base = S.ctl.ntie;
      for (uint32_t i = tid; i < mine; i += kThreads) {
        if (base + i < (uint32_t)kCap) {
          dsmem_st(dsmem_addr(&S.ckey[base + i], 0), S.ckey[i]);
          dsmem_st(dsmem_addr(&S.cpos[base + i], 0), (uint32_t)S.cpos[i]);
        }
      }
    } else if (tid == 0) {
      S.ctl.above_of[0] = S.ctl.above;
    }
    cluster_sync();  // B: CTA 0 holds every candidate
    if (rank == 0) {
      if (tid == 0) S.ctl.ntie = 0u;
      __syncthreads();
      // ---- CTA 0: digits 2 and 3 among the candidates, then the ties ----
      const uint32_t total = S.ctl.ccount;
      bool ok = total == eq1;  // every candidate arrived (else: slow path)
      uint32_t k_rem = (uint32_t)k_eff - above1;
      uint32_t T = 0u, need = 0u;
      if (ok) {
        for (uint32_t i = tid; i < total; i += kThreads)
          atomicAdd(&S.hloc[(S.ckey[i] >> kDigit3Bits) & (kBins2 - 1)], 1u);
        __syncthreads();
        find_digit<kBins2, kThreads>(S.hloc, k_rem, S.wsum, &S.found);
        const uint32_t d2 = S.found.digit;
        k_rem -= S.found.above;
        const uint32_t pre = (d1 << kDigit2Bits) | d2;
        for (uint32_t i = tid; i < total; i += kThreads)
          if ((S.ckey[i] >> kDigit3Bits) == pre) atomicAdd(&S.hacc3[S.ckey[i] & (kBins3 - 1)], 1u);
        __syncthreads();
        find_digit<kBins3, kThreads>(S.hacc3, k_rem, S.wsum, &S.found);
        T = (pre << kDigit3Bits) | S.found.digit;
        k_rem -= S.found.above;
        need = k_rem;  // ties on T to take, 1 <= need <= eq
        const uint32_t eq = S.found.eq;
        if (need < eq) {
          if (eq > (uint32_t)kMaxTies) {
            ok = false;
          } else {
            // the need-th lowest position among the ties
            for (uint32_t i = tid; i < total; i += kThreads)
              if (S.ckey[i] == T) S.tpos[atomicAdd(&S.ctl.ntie, 1u)] = S.cpos[i];
            __syncthreads();
            for (uint32_t j = tid; j < eq; j += kThreads) {
              const int pj = S.tpos[j];
              uint32_t r = 0u;
              for (uint32_t x = 0; x < eq; ++x) r += (S.tpos[x] < pj) ? 1u : 0u;
              if (r == need - 1u) S.ctl.tie_cut = pj;
            }
          }
        }
        __syncthreads();
      }
      if (ok) {
        // ---- mark the chosen candidates in their owners' bitmaps; count them per CTA ----
        const int cut = S.ctl.tie_cut;
        for (uint32_t i = tid; i < total; i += kThreads) {
          const uint32_t key = S.ckey[i];
          const int pos = S.cpos[i];
          if (key > T || (key == T && pos <= cut)) {
            const int owner = pos / chunk;
            const int lp = pos - owner * chunk;
            atomicAdd(&S.ctl.sel_of[owner], 1u);
            dsmem_red_or(dsmem_addr(&S.bm[lp >> 5], (uint32_t)owner), 1u << (lp & 31));
          }
        }
        __syncthreads();
        if (tid < C) {
          uint32_t base = 0u;
          for (int c = 0; c < tid; ++c) base += S.ctl.above_of[c] + S.ctl.sel_of[c];
          dsmem_st(dsmem_addr(&S.ctl.base, (uint32_t)tid), base);
          dsmem_st(dsmem_addr(&S.ctl.flag, (uint32_t)tid), kFast);
        }
      } else if (tid < C) {
        dsmem_st(dsmem_addr(&S.ctl.flag, (uint32_t)tid), kSlow);
      }
    }
    cluster_sync();  // C: results are in every CTA
  } else {
    // Too many candidates for the list: drain the copies issued above, then take the slow path.
    if (lane == 0)
      for (int j = 0; j < min(kSlots, my_tiles); ++j)
        if (!mbar_wait_bounded(&S.full[warp][j % kSlots], 0u)) waited_ok = false;
    __syncthreads();
    cluster_wait();
    if (C > 1 && rank == 0)
      for (int i = tid; i < kHistBins / 4; i += kThreads)
        reinterpret_cast<uint4*>(const_cast<uint32_t*>(ghist))[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tid == 0) S.ctl.flag = kSlow;
    __syncthreads();
  }

  uint32_t out_base;
  if (S.ctl.flag == kFast) {
    out_base = S.ctl.base;
  } else {
    // ------------------------------------------------------------ slow path: re-read the keys
    for (int i = tid; i < kBins2; i += kThreads) {
      S.hloc[i] = 0u;
      S.hacc2[i] = 0u;
    }
    for (int i = tid; i < kBins3; i += kThreads) S.hacc3[i] = 0u;
    if (tid == 0) S.found = Found{};
    cluster_sync();  // every CTA's accumulators are clear before the adds
    uint32_t k_rem = (uint32_t)k_eff - above1;
    // digit 2
    for (int i = tid; i < len; i += kThreads) {
      const uint32_t key = gk[i];
      if ((key >> kHistShift) == d1) atomicAdd(&S.hloc[(key >> kDigit3Bits) & (kBins2 - 1)], 1u);
    }
    __syncthreads();
    for (int i = tid; i < kBins2; i += kThreads)
      if (S.hloc[i]) dsmem_red_add(dsmem_addr(&S.hacc2[i], 0), S.hloc[i]);
    cluster_sync();
    find_digit<kBins2, kThreads>(cg::this_cluster().map_shared_rank(S.hacc2, 0), k_rem, S.wsum, &S.found);
    const uint32_t pre = (d1 << kDigit2Bits) | S.found.digit;
    k_rem -= S.found.above;
    // digit 3
    for (int i = tid; i < kBins3; i += kThreads) S.hloc[i] = 0u;
    __syncthreads();
    for (int i = tid; i < len; i += kThreads) {
      const uint32_t key = gk[i];
      if ((key >> kDigit3Bits) == pre) atomicAdd(&S.hloc[key & (kBins3 - 1)], 1u);
    }
    __syncthreads();
    for (int i = tid; i < kBins3; i += kThreads)
      if (S.hloc[i]) dsmem_red_add(dsmem_addr(&S.hacc3[i], 0), S.hloc[i]);
    cluster_sync();
    find_digit<kBins3, kThreads>(cg::this_cluster().map_shared_rank(S.hacc3, 0), k_rem, S.wsum, &S.found);
    const uint32_t T = (pre << kDigit3Bits) | S.found.digit;
    const uint32_t need = k_rem - S.found.above;
    // bits above T and ties on T, word by word; counts per CTA
    uint32_t n_above = 0u, n_tie = 0u;
    for (int w = w0; w < w1; ++w) {
      uint32_t ab = 0u, tb = 0u;
      for (int e = 0; e < 32 && w * 32 + e < len; ++e) {
        const uint32_t key = gk[w * 32 + e];
        ab |= (key > T ? 1u : 0u) << e;
        tb |= (key == T ? 1u : 0u) << e;
      }
      S.bm[w] = ab;
      S.ckey[w] = tb;
      n_above += (uint32_t)__popc(ab);
      n_tie += (uint32_t)__popc(tb);
    }
    uint32_t tot_above, tot_tie;
    const uint32_t tie_pre = block_excl_scan<kThreads>(n_tie, S.wsum, &tot_tie);
    block_excl_scan<kThreads>(n_above, S.wsum, &tot_above);
    if (tid == 0) {
      dsmem_st(dsmem_addr(&S.ctl.above_of[rank], 0), tot_above);
      dsmem_st(dsmem_addr(&S.ctl.tie_of[rank], 0), tot_tie);
    }
    cluster_sync();
    if (tid == 0) {
      uint32_t ties_before = 0u, base = 0u;
      for (int c = 0; c < (int)rank; ++c) {
        const uint32_t a = dsmem_ld(dsmem_addr(&S.ctl.above_of[c], 0));
        const uint32_t t = dsmem_ld(dsmem_addr(&S.ctl.tie_of[c], 0));
        const uint32_t taken = need > ties_before ? min(t, need - ties_before) : 0u;
        base += a + taken;
        ties_before += t;
      }
      S.ctl.base = base;
      S.ctl.ntie = ties_before;
    }
    cluster_sync();  // every CTA has read CTA 0's counts
    // take the ties in position order while the running tie rank is below need
    uint32_t r = S.ctl.ntie + tie_pre;
    for (int w = w0; w < w1; ++w) {
      uint32_t tb = S.ckey[w], take = 0u;
      while (tb) {
        const int e = __ffs(tb) - 1;
        tb &= tb - 1u;
        if (r < need) take |= 1u << e;
        ++r;
      }
      S.bm[w] |= take;
    }
    __syncthreads();
    out_base = S.ctl.base;
  }

  // ---------------------------------------------------------------- ordered output
  {
    uint32_t cnt = 0u;
    for (int w = w0; w < w1; ++w) cnt += (uint32_t)__popc(S.bm[w]);
    uint32_t tot;
    uint32_t o = out_base + block_excl_scan<kThreads>(cnt, S.wsum, &tot);
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = S.bm[w];
      while (bits) {
        const int e = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (o < (uint32_t)k_eff) idx[o] = c0 + w * 32 + e;
        ++o;
      }
    }
  }
  for (int j = k_eff + (int)rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = -1;
  if (!waited_ok) record_error(p.err, kDevWaitTimeout, (uint32_t)bh);
}

}  // namespace

bool plan_select(SelectParams& p, int num_sms) {
  const int heads = p.B * p.Hkv;
  // One CTA per SM.  Split a head over a cluster while its chunk is too long, and while the
  // grid still leaves SMs idle (up to the portable cluster size).
  int C = 1;
  while (C < kMaxCluster && (p.cap + C - 1) / C > kChunkMax) C *= 2;
  while (C < 8 && (long)heads * C * 2 <= (long)num_sms) C *= 2;
  if ((p.cap + C - 1) / C > kChunkMax) return false;
  p.cluster = C;
  p.chunk = (((p.cap + C - 1) / C) + 31) & ~31;
  p.cand_cap = kCap;
  p.off_hist = 0;
  p.off_ctl = 0;
  p.threads = C >= 2 ? 512 : 1024;
  p.smem_bytes = p.threads == 512 ? (int)sizeof(SelSmem<512>) : (int)sizeof(SelSmem<1024>);
  return true;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  auto kern = p.threads == 512 ? select_topk_kernel<512> : select_topk_kernel<1024>;
  const cudaError_t e = prepare_kernel((const void*)kern, p.smem_bytes, p.cluster > 8);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)p.cluster, (unsigned)(p.B * p.Hkv), 1), dim3((unsigned)p.threads),
                    (size_t)p.smem_bytes, stream, p, (unsigned)p.cluster);
}

}  // namespace sas
