// Fused score scan + per-KV-head top-k selection (sm_100a).
//
// One thread-block cluster per (sequence b, KV head h).  Each CTA of the cluster owns a
// contiguous chunk of positions:
//   1. q-bar = mean of the G query heads of h, q-hat = sigma * M[h] q-bar (JSSA page, section
//      打分误差的定义: selection uses the group-mean query and s-hat = q-bar^T M^T M k).
//   2. The chunk's projected-cache rows stream through a ring of shared-memory stages filled by
//      bulk copies on the TMA engine (one copy per contiguous run: the whole stage for the
//      contiguous layout, one per 64-token page for the paged one).  Each thread scores one
//      row: u_i = q-hat . Kproj_i (+ lambda log g_i, SAS page section 2.1), with packed fp32
//      FMAs, and stores the order-preserving uint32 key of u_i in shared memory.  Scoring scans
//      every candidate (JSSA page, section Triton 内核的三个设计点: scoring is not sparse).
//   3. Radix select of the k-th largest key over the whole cluster: up to three digit passes
//      (11, 11, 10 bits).  Each CTA histograms its chunk in shared memory, adds the non-zero
//      bins into rank 0's histogram through distributed shared memory, rank 0 finds the digit
//      holding the k-th key and broadcasts it.  A pass that isolates exactly the remaining
//      count ends the search early.
//   4. Ordered compaction: positions with a larger key are selected, and of those with the
//      threshold key the lowest positions fill the remainder (exact ties -> lower position).
//      A cluster-wide exclusive count gives every position its output slot, so the index list
//      comes out in ascending order with no sort.
// Scores never leave the chip.  The per-KV-head top-k shared by the G query heads is the
// selection rule of the JSSA page, section JSSA 的整体结构 / Figure 1.
#include <cooperative_groups.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace cg = cooperative_groups;

namespace sas {
namespace {

constexpr int kThreads = 256;
constexpr int kStageRows = 256;  // one row per thread per stage
constexpr int kBins = 2048;      // 11-bit digits
constexpr int kMaxStages = 8;

struct Ctl {
  uint32_t prefix, mask, k_rem, eq;
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

template <int R>
__global__ void __launch_bounds__(kThreads) select_topk_kernel(const SelectParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int C = (int)cluster.num_blocks();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;

  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  unsigned char* ring = smem + p.off_ring;
  uint32_t* hist_local = reinterpret_cast<uint32_t*>(ring);
  uint32_t* hist_global = hist_local + kBins;
  float* qbar = reinterpret_cast<float*>(smem + p.off_q);
  float* qhat = qbar + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + p.off_ctl);
  uint32_t* wsum = reinterpret_cast<uint32_t*>(ctl + 1);

  // ---- per-sequence values (checked on the device) ----
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (rank == 0 && tid == 0 && h == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    n = 0;
  }
  int kb = p.kvec[b];
  if (kb > p.k_max) {
    if (rank == 0 && tid == 0 && h == 0) record_error(p.err, kDevKOverMax, (uint32_t)b);
    kb = p.k_max;
  }
  const int k_eff = max(0, min(kb, n));
  int32_t* idx = p.idx_out + (size_t)bh * p.k_max;

  // Nothing to rank: empty selection, or every position selected (scores still computed when
  // they are requested).  Uniform per cluster.
  const bool want_scores = (p.scores_out != nullptr) && n > 0;
  if (!want_scores && (k_eff == 0 || k_eff == n)) {
    for (int j = rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = (j < k_eff) ? j : -1;
    return;
  }

  // ---- this CTA's positions [c0, c1) ----
  const int chunk_b = ((n + C - 1) / C + 511) & ~511;  // multiple of 512 -> even run
  const int run = chunk_b / kThreads;                  // positions per thread in the select
  const int c0 = min(rank * chunk_b, n);
  const int c1 = min(c0 + chunk_b, n);
  const int len = c1 - c0;

  // ---- 1. q-bar and q-hat ----
  for (int c = tid; c < p.d; c += kThreads) {
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + (size_t)h * p.G) * p.d + c;
    float s = 0.f;
    for (int g = 0; g < p.G; ++g) s += __bfloat162float(qg[(size_t)g * p.d]);
    qbar[c] = s / (float)p.G;
  }
  if (tid == 0) {
    for (int s = 0; s < p.nstages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  for (int j = warp; j < R; j += kThreads / 32) {
    const float* Mj = p.M + ((size_t)h * R + j) * p.d;
    float s = 0.f;
    for (int c = lane; c < p.d; c += 32) s = fmaf(Mj[c], qbar[c], s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) qhat[j] = s * p.sigma;
  }
  __syncthreads();

  // Each thread reads its row's 16-byte chunks in a rotated order so that the 8 lanes of a
  // shared-memory phase hit distinct banks; q-hat is held in the same rotated order, so the
  // register index stays static.
  constexpr int CPR = R / 8;                        // 16-byte chunks per row
  constexpr int STAG = (64 / R) > 1 ? (64 / R) : 1; // lanes sharing a rotation
  const int rot = (tid / STAG) % CPR;
  float2 qr[CPR][4];
#pragma unroll
  for (int cc = 0; cc < CPR; ++cc) {
    const int ch = (cc + rot) % CPR;
#pragma unroll
    for (int e = 0; e < 4; ++e) qr[cc][e] = make_float2(qhat[ch * 8 + 2 * e], qhat[ch * 8 + 2 * e + 1]);
  }

  // ---- 2. stream the chunk's projected rows ----
  const bool gated = (p.log_g != nullptr);
  const size_t lg_base = (size_t)bh * p.cap;
  const int nst = (len + kStageRows - 1) / kStageRows;
  const int kp_stage_bytes = kStageRows * R * 2;

  auto issue = [&](int s) {
    const int r0 = s * kStageRows;
    const int nr = min(kStageRows, len - r0);
    const int slot = s % p.nstages;
    unsigned char* dst = ring + (size_t)slot * p.stage_bytes;
    const int pos0 = c0 + r0;
    uint32_t bytes = 0;
    if (!p.paged) {
      bytes += (uint32_t)nr * R * 2;
    } else {
      for (int t = 0; t < nr; t += 64) {
        const int pg = p.page_table[(size_t)b * p.max_pages + (pos0 + t) / 64];
        if (pg >= 0 && pg < p.num_pages) bytes += (uint32_t)min(64, nr - t) * R * 2;
      }
    }
    if (gated) bytes += (uint32_t)((nr + 3) & ~3) * 4;
    mbar_arrive_expect_tx(&bars[slot], bytes);
    if (!p.paged) {
      const __nv_bfloat16* src = p.kproj + ((size_t)bh * p.cap + pos0) * R;
      bulk_g2s(dst, src, (uint32_t)nr * R * 2, &bars[slot]);
    } else {
      for (int t = 0; t < nr; t += 64) {
        const int pos = pos0 + t;
        const int pg = p.page_table[(size_t)b * p.max_pages + pos / 64];
        if (pg >= 0 && pg < p.num_pages) {
          const __nv_bfloat16* src = p.kproj + (((size_t)pg * p.Hkv + h) * 64 + (pos & 63)) * R;
          bulk_g2s(dst + (size_t)t * R * 2, src, (uint32_t)min(64, nr - t) * R * 2, &bars[slot]);
        } else {
          record_error(p.err, kDevBadPage, (uint32_t)b);
        }
      }
    }
    if (gated) bulk_g2s(dst + kp_stage_bytes, p.log_g + lg_base + pos0, (uint32_t)((nr + 3) & ~3) * 4, &bars[slot]);
  };

  if (tid == 0)
    for (int s = 0; s < min(nst, p.nstages); ++s) issue(s);

  bool waited_ok = true;
  for (int s = 0; s < nst; ++s) {
    const int slot = s % p.nstages;
    const uint32_t parity = (uint32_t)(s / p.nstages) & 1u;
    if (!mbar_wait_bounded(&bars[slot], parity)) waited_ok = false;
    const int row = s * kStageRows + tid;
    if (row < len) {
      const unsigned char* st = ring + (size_t)slot * p.stage_bytes;
      const uint4* kr = reinterpret_cast<const uint4*>(st + (size_t)tid * (R * 2));
      // Per-chunk partial sums, combined by a butterfly over the chunk index: the result is
      // the same for every rotation, so identical rows give bit-identical scores (exact ties).
      float pc[CPR];
#pragma unroll
      for (int cc = 0; cc < CPR; ++cc) {
        const uint4 w = kr[(cc + rot) % CPR];
        float2 a = ffma2(qr[cc][0], make_float2(bf16lo(w.x), bf16hi(w.x)), make_float2(0.f, 0.f));
        a = ffma2(qr[cc][1], make_float2(bf16lo(w.y), bf16hi(w.y)), a);
        a = ffma2(qr[cc][2], make_float2(bf16lo(w.z), bf16hi(w.z)), a);
        a = ffma2(qr[cc][3], make_float2(bf16lo(w.w), bf16hi(w.w)), a);
        pc[cc] = a.x + a.y;
      }
#pragma unroll
      for (int half = CPR / 2; half >= 1; half >>= 1)
#pragma unroll
        for (int cc = 0; cc < half; ++cc) pc[cc] = pc[cc] + pc[cc + half];
      float u = pc[0];
      if (gated) {
        const float lg = reinterpret_cast<const float*>(st + kp_stage_bytes)[tid];
        u = fmaf(p.lam, lg, u);
      }
      keys[row + row / run] = float_key(u);
      if (p.scores_out != nullptr) p.scores_out[lg_base + c0 + row] = u;
    }
    __syncthreads();
    if (tid == 0 && s + p.nstages < nst) issue(s + p.nstages);
  }
  if (!waited_ok) record_error(p.err, kDevWaitTimeout, (uint32_t)bh);

  if (k_eff == 0) {  // scores were requested, nothing is selected (uniform per cluster)
    for (int j = rank * kThreads + tid; j < p.k_max; j += C * kThreads) idx[j] = -1;
    return;
  }

  // ---- 3. radix select across the cluster ----
  for (int i = tid; i < 2 * kBins; i += kThreads) hist_local[i] = 0u;
  cluster.sync();  // all keys written; every CTA's histograms zeroed

  uint32_t prefix = 0u, mask = 0u, k_rem = (uint32_t)k_eff;
  const int my0 = tid * run;
  uint32_t* g0 = cluster.map_shared_rank(hist_global, 0);
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3ffu : 0x7ffu;
    const int nb = (int)dmask + 1;
    if (pass > 0) {
      for (int i = tid; i < kBins; i += kThreads) hist_local[i] = 0u;
      __syncthreads();
    }
    for (int i = 0; i < run; ++i) {
      const int li = my0 + i;
      uint32_t key = 0u;
      bool act = false;
      if (li < len) {
        key = keys[li + tid];  // == keys[li + li / run]
        act = (key & mask) == prefix;
      }
      hist_add(hist_local, (key >> shift) & dmask, act);
    }
    __syncthreads();
    for (int i = tid; i < nb; i += kThreads) {
      const uint32_t v = hist_local[i];
      if (v) atomicAdd(&g0[i], v);
    }
    cluster.sync();
    if (rank == 0) {
      const int per = nb / kThreads;
      const int hi = nb - tid * per;  // thread t covers digits [hi - per, hi), highest first
      uint32_t tsum = 0u;
      for (int j = 1; j <= per; ++j) tsum += hist_global[hi - j];
      uint32_t tot;
      const uint32_t above = block_excl_scan(tsum, wsum, &tot);
      if (above < k_rem && k_rem <= above + tsum) {
        uint32_t a = above;
        for (int j = 1; j <= per; ++j) {
          const uint32_t c = hist_global[hi - j];
          if (a + c >= k_rem) {
            const uint32_t digit = (uint32_t)(hi - j);
            Ctl v;
            v.prefix = prefix | (digit << shift);
            v.mask = mask | (dmask << shift);
            v.k_rem = k_rem - a;
            v.eq = c;
            for (int rr = 0; rr < C; ++rr) {
              Ctl* dstc = cluster.map_shared_rank(ctl, rr);
              dstc->prefix = v.prefix;
              dstc->mask = v.mask;
              dstc->k_rem = v.k_rem;
              dstc->eq = v.eq;
            }
            break;
          }
          a += c;
        }
      }
      __syncthreads();
      for (int i = tid; i < nb; i += kThreads) hist_global[i] = 0u;
    }
    cluster.sync();
    prefix = ctl->prefix;
    mask = ctl->mask;
    k_rem = ctl->k_rem;
    if (ctl->eq == k_rem) break;  // the threshold digit holds exactly the remainder
  }

  // ---- 4. ordered compaction ----
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
  if (tid == 0) {
    uint32_t gb = 0u, eb = 0u;
    for (int rr = 0; rr < rank; ++rr) {
      const Ctl* rc = cluster.map_shared_rank(ctl, rr);
      gb += rc->cta_gt;
      eb += rc->cta_eq;
    }
    ctl->gt_before = gb;
    ctl->eq_before = eb;
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
  cluster.sync();  // peers may still read this CTA's control block
}

template <int R>
cudaError_t launch_r(const SelectParams& p, cudaStream_t stream) {
  auto kern = select_topk_kernel<R>;
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
  if (p.r != 16 && p.r != 32 && p.r != 64) return false;
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
  p.stage_bytes = kStageRows * p.r * 2 + kStageRows * 4;
  const int keys_bytes = ((chunk + kThreads) * 4 + 127) & ~127;
  // Ring depth: deeper when few CTAs share an SM.
  const long ctas = (long)heads * C;
  int ns = ctas <= num_sms ? 6 : (ctas <= 2L * num_sms ? 4 : 2);
  if (ns > kMaxStages) ns = kMaxStages;
  p.nstages = ns;
  int ring = ns * p.stage_bytes;
  if (ring < 2 * kBins * 4) ring = 2 * kBins * 4;
  ring = (ring + 127) & ~127;
  p.off_ring = keys_bytes;
  p.off_q = p.off_ring + ring;
  p.off_bar = p.off_q + (128 + 64) * 4;
  p.off_ctl = p.off_bar + kMaxStages * 8;
  p.smem_bytes = p.off_ctl + (int)sizeof(Ctl) + (kThreads / 32) * 4;
  return p.smem_bytes <= 227 * 1024;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  switch (p.r) {
    case 16: return launch_r<16>(p, stream);
    case 32: return launch_r<32>(p, stream);
    case 64: return launch_r<64>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sas
