// Gather-free split-K decode attention over per-KV-head index sets (sm_100a).
//
// JSSA page, section 原理详解(二) / Triton 内核的三个设计点: one launch per layer serves
// every KV head, each query head is mapped to the index set its KV head selected, and the K/V
// rows are read where they live, with no staging copy of the selected cache.  One token's K
// (or V) head slice is contiguous (section 不规则索引本身不是障碍): the lanes of a warp copy
// the selected rows in 16-byte pieces (cp.async) straight into the warp's shared-memory ring;
// the page holding each row is resolved per index for the paged layout.  The dense variant
// fetches whole 8-row tiles with one bulk copy (TMA engine) each for K and V.
//
// Grid: (splits, B*Hkv, G/gt).  A CTA takes a contiguous slice of one (b, h) index list and
// gt query heads of h; its 4 warps take 8-token tiles of the slice in turn, each warp with its
// own ring of stages and its own online-softmax state (running max m, sum l, accumulator), in
// fp32.  Logits z = sigma q.K_i (+ lambda log g_i, SAS page section 2.1).  The warps merge in
// shared memory and the CTA writes one partial (m, l, acc) per query head to the workspace; a
// second kernel, one CTA per (b, h, head group) (four, each with a quarter of the channels,
// when head groups are few), merges the splits in split order (deterministic) and writes the
// output.  The split CTAs wait on no counter or fence, so each
// frees its SM slot as soon as its partial is written.  The dense variant (idx = 0..N_b-1) is
// the full-KV baseline.
#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 8;     // tokens per warp tile
constexpr int kStages = 2;   // ring depth per warp

// 16-byte global -> shared copy by this thread (completes at the next wait on its group).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D, int GT>
struct Geo {
  static constexpr int LPR = D / 8;            // lanes per K row (16 bytes each)
  static constexpr int RPI = 32 / LPR;         // rows per warp instruction
  static constexpr int NP = kTile / RPI;       // row groups per lane per tile
  static constexpr int NV = NP * GT;           // partial dot products per lane per tile
  static constexpr int CPL = D / 32;           // output channels per lane (PV)
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int STAGE_BYTES = 2 * kTile * ROW_BYTES;
  static constexpr int LOG_LPR = (LPR == 16) ? 4 : 3;
  static constexpr int LOG_NV = (NV >= 16) ? 4 : (NV == 8 ? 3 : (NV == 4 ? 2 : (NV == 2 ? 1 : 0)));
  // After the reduction a lane's value index is (lane % LPR) >> SHIFT (SHIFT > 0 when NV < LPR).
  static constexpr int SHIFT = LOG_LPR > LOG_NV ? LOG_LPR - LOG_NV : 0;
  static constexpr int LOG_GT = GT == 4 ? 2 : (GT == 2 ? 1 : 0);
};

struct Smem {
  int off_rows, off_lg, off_ring, off_pbuf, off_sbuf, off_merge, off_bars, total;
};

// The gate terms' buffer (lg) is laid out only for the gated variant.
template <int D, int GT>
__host__ __device__ inline Smem smem_layout(int split_len, int splits, bool with_lg) {
  using Gm = Geo<D, GT>;
  Smem s;
  int o = 0;
  s.off_rows = o;  o += split_len * 4;
  s.off_lg = o;    o += with_lg ? split_len * 4 : 0;
  o = (o + 127) & ~127;
  s.off_ring = o;
  // After the tile loop the ring is idle: the warp merge (and the split merge) reuse it.
  const int ring = kWarps * kStages * Gm::STAGE_BYTES;
  const int merge = kWarps * GT * (D + 2) * 4;
  s.off_merge = o;
  o += ring > merge ? ring : merge;
  s.off_pbuf = o;  o += kWarps * kTile * GT * 4;
  s.off_sbuf = o;  o += kWarps * GT * 4;
  o = (o + 7) & ~7;
  s.off_bars = o;  o += kWarps * kStages * 8;
  s.total = o;
  return s;
}

template <int D, int GT, bool GATED, bool PAGED, bool DENSE>
__global__ void __launch_bounds__(kThreads) attend_kernel(const AttendParams p) {
  using Gm = Geo<D, GT>;
  extern __shared__ __align__(128) unsigned char smem[];
  const Smem L = smem_layout<D, GT>(p.split_len, p.splits, GATED);
  uint32_t* rows_s = reinterpret_cast<uint32_t*>(smem + L.off_rows);
  float* lg_s = reinterpret_cast<float*>(smem + L.off_lg);
  unsigned char* ring = smem + L.off_ring;
  float* pbuf_all = reinterpret_cast<float*>(smem + L.off_pbuf);
  float* sbuf_all = reinterpret_cast<float*>(smem + L.off_sbuf);
  float* merge = reinterpret_cast<float*>(smem + L.off_merge);
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(smem + L.off_bars);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int gz = blockIdx.z;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int bhz = bh * p.ngz + gz;

  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (split == 0 && tid == 0 && h == 0 && gz == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    n = 0;
  }
  int count = n;
  if (!DENSE) {
    int kb = p.kvec[b];
    kb = min(kb, p.k_max);
    count = max(0, min(kb, n));
  }
  const int j0 = split * p.split_len;
  const int j1 = min(j0 + p.split_len, count);
  const int cnt = max(0, j1 - j0);

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars_all[warp * kStages + s], 1);
    fence_barrier_init();
  }

  // ---- query slice in registers: lane holds channels c0..c0+7 of each of its gt heads ----
  const int rl = lane % Gm::LPR;   // lane within its row
  const int rs = lane / Gm::LPR;   // row slot within a warp instruction
  const int c0 = rl * 8;
  float2 qv[GT][4];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    const int hq = h * p.G + gz * GT + g;
    const uint4 w = *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + hq) * D + c0);
    qv[g][0] = make_float2(bf16lo(w.x) * p.sigma, bf16hi(w.x) * p.sigma);
    qv[g][1] = make_float2(bf16lo(w.y) * p.sigma, bf16hi(w.y) * p.sigma);
    qv[g][2] = make_float2(bf16lo(w.z) * p.sigma, bf16hi(w.z) * p.sigma);
    qv[g][3] = make_float2(bf16lo(w.w) * p.sigma, bf16hi(w.w) * p.sigma);
  }
  // The index list (written by the selection) and the workspace are read only from here on.
  pdl_wait();
  pdl_trigger();

  // ---- resolve the slice's rows (and gate terms) once; loads batched 4 per thread ----
  for (int jb = 0; jb < cnt; jb += 4 * kThreads) {
    int iv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * kThreads + tid;
      iv[u] = (j < cnt) ? (DENSE ? (j0 + j) : p.idx[(size_t)bh * p.k_max + j0 + j]) : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!DENSE && (iv[u] < 0 || iv[u] >= n)) {
        record_error(p.err, kDevBadIndex, (uint32_t)bh);
        iv[u] = 0;
      }
    }
    int pg[4] = {0, 0, 0, 0};
    float lgv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * kThreads + tid;
      if (j < cnt) {
        if (PAGED) pg[u] = p.page_table[(size_t)b * p.max_pages + (iv[u] >> 6)];
        if (GATED) lgv[u] = p.log_g[(size_t)bh * p.cap + iv[u]];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * kThreads + tid;
      if (j < cnt) {
        uint32_t row;
        if (PAGED) {
          int g = pg[u];
          if (g < 0 || g >= p.num_pages) {
            record_error(p.err, kDevBadPage, (uint32_t)b);
            g = 0;
          }
          row = ((uint32_t)g * (uint32_t)p.Hkv + (uint32_t)h) * 64u + (uint32_t)(iv[u] & 63);
        } else {
          row = (uint32_t)bh * (uint32_t)p.cap + (uint32_t)iv[u];
        }
        rows_s[j] = row;
        if (GATED) lg_s[j] = p.lam * lgv[u];
      }
    }
  }
  __syncthreads();

  // This lane's logit slot after the reduction: value index vi -> (row group, head).
  const int vi = rl >> Gm::SHIFT;
  const int my_rg = vi / GT;
  const int my_g = vi % GT;
  const int my_tl = my_rg * Gm::RPI + rs;  // token within the tile
  const bool owner = (rl & ((1 << Gm::SHIFT) - 1)) == 0;

  unsigned char* wring = ring + (size_t)warp * kStages * Gm::STAGE_BYTES;
  uint64_t* bars = bars_all + warp * kStages;
  float* pbuf = pbuf_all + warp * kTile * GT;
  float* sbuf = sbuf_all + warp * GT;

  const int ntiles = (cnt + kTile - 1) / kTile;
  const int nt_w = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;

  // Tile `it` of this warp into its ring slot.  Dense: a tile is 8 consecutive positions
  // starting at a multiple of 8, i.e. consecutive rows of the cache (within one 64-token page
  // for the paged layout), fetched as one bulk copy each for K and V.  Sparse: the selected
  // rows are scattered, so every lane copies 16-byte pieces of them (cp.async, one group per
  // tile; an empty group past the last tile keeps the group count uniform).
  constexpr int kPieces = kTile * D / 8;          // 16-byte pieces of the tile's K rows
  constexpr int kPiecesPerLane = kPieces / 32;
  auto issue = [&](int it) {
    const int slot = it % kStages;
    unsigned char* st = wring + (size_t)slot * Gm::STAGE_BYTES;
    if (DENSE) {
      const int tile = warp + it * kWarps;
      const int tb = tile * kTile;
      const int ntok = min(kTile, cnt - tb);
      if (lane == 0) mbar_arrive_expect_tx(&bars[slot], (uint32_t)(ntok * 2 * Gm::ROW_BYTES));
      __syncwarp();
      if (lane < 2) {
        const uint32_t row = rows_s[tb];
        const __nv_bfloat16* src = (lane ? p.V : p.K) + (size_t)row * D;
        bulk_g2s(st + (size_t)(lane ? kTile : 0) * Gm::ROW_BYTES, src, (uint32_t)(ntok * Gm::ROW_BYTES), &bars[slot]);
      }
    } else {
      if (it < nt_w) {
        const int tb = (warp + it * kWarps) * kTile;
        const int ntok = min(kTile, cnt - tb);
#pragma unroll
        for (int i = 0; i < kPiecesPerLane; ++i) {
          const int c = lane + 32 * i;         // piece c: row c / (D/8), part c % (D/8)
          const int t = c / (D / 8), part = c % (D / 8);
          if (t < ntok) {
            const size_t row = rows_s[tb + t];
            cp_async16(st + (size_t)t * Gm::ROW_BYTES + part * 16, p.K + row * D + part * 8);
            cp_async16(st + (size_t)(kTile + t) * Gm::ROW_BYTES + part * 16, p.V + row * D + part * 8);
          }
        }
      }
      cp_async_commit();
    }
  };

  for (int it = 0; it < (DENSE ? min(kStages, nt_w) : kStages); ++it) issue(it);

  float m_run = -INFINITY;  // running max of this lane's head
  float l_part = 0.f;       // this lane's share of the running sum (owner lanes)
  float acc[GT][Gm::CPL];
#pragma unroll
  for (int g = 0; g < GT; ++g)
#pragma unroll
    for (int c = 0; c < Gm::CPL; ++c) acc[g][c] = 0.f;
  bool waited_ok = true;

  for (int it = 0; it < nt_w; ++it) {
    const int slot = it % kStages;
    const int tb = (warp + it * kWarps) * kTile;
    const int ntok = min(kTile, cnt - tb);
    if (DENSE) {
      if (!mbar_wait_bounded(&bars[slot], (uint32_t)(it / kStages) & 1u)) waited_ok = false;
    } else {
      cp_async_wait<kStages - 1>();  // this lane's pieces of tile `it` have landed
      __syncwarp();                  // ... and every other lane's
    }
    const unsigned char* st = wring + (size_t)slot * Gm::STAGE_BYTES;

    // QK: partial dots of this lane's 8 channels, for NP rows x GT heads.
    float v[Gm::NV];
#pragma unroll
    for (int rg = 0; rg < Gm::NP; ++rg) {
      const int tl = rg * Gm::RPI + rs;
      const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)tl * Gm::ROW_BYTES + c0 * 2);
      const float2 k0 = make_float2(bf16lo(w.x), bf16hi(w.x));
      const float2 k1 = make_float2(bf16lo(w.y), bf16hi(w.y));
      const float2 k2 = make_float2(bf16lo(w.z), bf16hi(w.z));
      const float2 k3 = make_float2(bf16lo(w.w), bf16hi(w.w));
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float2 a = make_float2(0.f, 0.f);
        a = ffma2(qv[g][0], k0, a);
        a = ffma2(qv[g][1], k1, a);
        a = ffma2(qv[g][2], k2, a);
        a = ffma2(qv[g][3], k3, a);
        v[rg * GT + g] = a.x + a.y;
      }
    }
    // Reduce over the LPR lanes of each row: transposing butterfly, then plain butterfly.
#pragma unroll
    for (int lvl = 0; lvl < Gm::LOG_LPR; ++lvl) {
      const int m = Gm::LPR >> (lvl + 1);
      if (lvl < Gm::LOG_NV) {
        const int half = Gm::NV >> (lvl + 1);
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
      }
    }
    float z = v[0];
    if (GATED) z += lg_s[tb + min(my_tl, ntok - 1)];
    if (my_tl >= ntok) z = -INFINITY;

    // Online softmax for head my_g: max over the lanes holding the same head.
    float tmax = z;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      // skip lane bits that encode the head (bits SHIFT .. SHIFT+LOG_GT-1 of rl)
      const bool head_bit = (m >= (1 << Gm::SHIFT)) && (m < (1 << (Gm::SHIFT + Gm::LOG_GT)));
      if (!head_bit) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
    }
    const float m_new = fmaxf(m_run, tmax);
    const float scale = (m_new == -INFINITY) ? 1.f : __expf(m_run - m_new);
    const float pz = (m_new == -INFINITY) ? 0.f : __expf(z - m_new);
    m_run = m_new;
    if (owner) {
      l_part = l_part * scale + pz;
      if (my_tl < ntok) pbuf[my_tl * GT + my_g] = pz;
      if (my_tl == 0) sbuf[my_g] = scale;
    }
    __syncwarp();

    // PV: lane owns channels lane*CPL .. +CPL-1 of every head.
    float sc[GT];
#pragma unroll
    for (int g = 0; g < GT; ++g) sc[g] = sbuf[g];
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int c = 0; c < Gm::CPL; ++c) acc[g][c] *= sc[g];
    const unsigned char* vst = st + (size_t)kTile * Gm::ROW_BYTES;
    for (int tl = 0; tl < ntok; ++tl) {
      float pw[GT];
#pragma unroll
      for (int g = 0; g < GT; ++g) pw[g] = pbuf[tl * GT + g];
      if constexpr (Gm::CPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vst + (size_t)tl * Gm::ROW_BYTES + lane * 8);
        const float2 v0 = make_float2(bf16lo(w.x), bf16hi(w.x));
        const float2 v1 = make_float2(bf16lo(w.y), bf16hi(w.y));
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float2 pp = make_float2(pw[g], pw[g]);
          float2 a01 = ffma2(pp, v0, make_float2(acc[g][0], acc[g][1]));
          float2 a23 = ffma2(pp, v1, make_float2(acc[g][2], acc[g][3]));
          acc[g][0] = a01.x; acc[g][1] = a01.y; acc[g][2] = a23.x; acc[g][3] = a23.y;
        }
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(vst + (size_t)tl * Gm::ROW_BYTES + lane * 4);
        const float2 v0 = make_float2(bf16lo(w), bf16hi(w));
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float2 pp = make_float2(pw[g], pw[g]);
          float2 a01 = ffma2(pp, v0, make_float2(acc[g][0], acc[g][1]));
          acc[g][0] = a01.x; acc[g][1] = a01.y;
        }
      }
    }
    __syncwarp();
    if (DENSE) {
      if (it + kStages < nt_w) issue(it + kStages);
    } else {
      issue(it + kStages);
    }
  }
  if (!DENSE) cp_async_wait<0>();
  if (!waited_ok) record_error(p.err, kDevWaitTimeout, (uint32_t)bh);

  // ---- per-warp totals: l over the owner lanes of each head ----
  float l_tot = owner ? l_part : 0.f;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool head_bit = (m >= (1 << Gm::SHIFT)) && (m < (1 << (Gm::SHIFT + Gm::LOG_GT)));
    if (!head_bit) l_tot += __shfl_xor_sync(0xffffffffu, l_tot, m);
  }
  // The merge buffer aliases the ring: every warp must be done with its stages (all issued
  // copies have been waited for) before any warp writes its totals.
  __syncthreads();
  // merge: acc [warp][g][D] (16-byte rows of lanes), then (m, l) [warp][g][2]
  float* mml = merge + kWarps * GT * D;
  float* mw = merge + (size_t)warp * GT * D;
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    if constexpr (Gm::CPL == 4) {
      *reinterpret_cast<float4*>(mw + g * D + lane * 4) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    } else {
      *reinterpret_cast<float2*>(mw + g * D + lane * 2) = make_float2(acc[g][0], acc[g][1]);
    }
  }
  if (owner && my_tl == 0) {
    mml[(warp * GT + my_g) * 2] = m_run;
    mml[(warp * GT + my_g) * 2 + 1] = l_tot;
  }
  __syncthreads();

  // ---- CTA partial for this split: acc [GT][D] and (m, l) [GT][2] ----
  // Per head: M = max over the warps of m, weights f_w = exp(m_w - M) (0 for an empty warp),
  // L = sum f_w l_w; then acc = sum f_w acc_w, four channels per thread and step.
  const size_t nheads = (size_t)p.B * p.Hkv * p.ngz;
  float* pacc = p.partials + ((size_t)bhz * p.splits + split) * GT * D;
  float* pml = p.partials + nheads * p.splits * GT * D + ((size_t)bhz * p.splits + split) * GT * 2;
  float* cw = pbuf_all;   // [kWarps][GT] weights, then [GT] M (the tile buffers are idle now)
  if (tid < GT) {
    const int g = tid;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mml[(w * GT + g) * 2]);
    float Lc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mwv = mml[(w * GT + g) * 2];
      const float f = (M == -INFINITY || mwv == -INFINITY) ? 0.f : __expf(mwv - M);
      cw[w * GT + g] = f;
      Lc += f * mml[(w * GT + g) * 2 + 1];
    }
    cw[kWarps * GT + g] = M;
    pml[g * 2] = M;
    pml[g * 2 + 1] = Lc;
  }
  __syncthreads();
  for (int e = tid; e < GT * D / 4; e += kThreads) {
    const int g = (e * 4) / D;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (cw[kWarps * GT + g] != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = cw[w * GT + g];
        const float4 a = *reinterpret_cast<const float4*>(merge + (size_t)w * GT * D + e * 4);
        v.x += f * a.x;
        v.y += f * a.y;
        v.z += f * a.z;
        v.w += f * a.w;
      }
    }
    *reinterpret_cast<float4*>(pacc + e * 4) = v;
  }
}



// Merge of each head group's split partials, in split order (deterministic), and the output.
// Launched after the split kernel on the same stream with programmatic dependent launch: its
// wait returns once every split CTA has finished and its partial is visible.  NQ CTAs share a
// head group, each taking D / NQ of its channels (NQ = 4 when there are few head groups, so that
// more SMs read the partials and each warp has fewer loads in flight to wait for).
template <int D, int GT, int NQ>
__host__ __device__ inline int combine_smem_floats(int splits) {
  return ((splits * GT + GT + 3) & ~3) + kWarps * GT * (D / NQ);
}

template <int D, int GT, int NQ>
__global__ void __launch_bounds__(kThreads) combine_kernel(const AttendParams p) {
  constexpr int DC = D / NQ;                   // channels of this CTA
  extern __shared__ __align__(16) float csm[];
  float* wts = csm;                                          // [splits][GT] weights, [GT] 1/L
  float* red = csm + ((p.splits * GT + GT + 3) & ~3);       // [kWarps][GT * DC] warp sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bhz = blockIdx.x;
  const int c_base = blockIdx.y * DC;
  const int bh = bhz / p.ngz, gz = bhz % p.ngz;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const size_t nheads = (size_t)p.B * p.Hkv * p.ngz;
  pdl_wait();
  pdl_trigger();
  const float* bacc = p.partials + (size_t)bhz * p.splits * GT * D;
  const float* bml = p.partials + nheads * p.splits * GT * D + (size_t)bhz * p.splits * GT * 2;

  // Warp w sums splits w, w + 4, ... in order, kU splits per step with all their loads in flight;
  // lane owns OPL consecutive outputs (one head).  The first step's loads are issued before the
  // weights are computed, so the two reads of the partials overlap.
  constexpr int OPL = GT * DC / 32;
  static_assert(OPL >= 2 && OPL % 2 == 0, "two or more outputs per lane");
  constexpr int VW = (OPL % 4 == 0) ? 4 : 2;   // floats per load
  constexpr int kU = OPL <= 4 ? 8 : 4;         // splits per step (registers: kU * OPL)
  const int e0 = lane * OPL;
  const int gl = e0 / DC;
  const int coff = gl * D + c_base + e0 % DC;  // offset of the lane's outputs in a [GT][D] partial
  float va[kU][OPL];
  auto load_step = [&](int s0) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int s = s0 + u * kWarps;
      if (s < p.splits) {
        const float* a = bacc + (size_t)s * GT * D + coff;
#pragma unroll
        for (int i = 0; i < OPL; i += VW) {
          if constexpr (VW == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(a + i));
            va[u][i] = x.x; va[u][i + 1] = x.y; va[u][i + 2] = x.z; va[u][i + 3] = x.w;
          } else {
            const float2 x = __ldcg(reinterpret_cast<const float2*>(a + i));
            va[u][i] = x.x; va[u][i + 1] = x.y;
          }
        }
      }
    }
  };
  load_step(warp);

  if (warp < GT) {
    const int g = warp;
    float M = -INFINITY;
    for (int s = lane; s < p.splits; s += 32) M = fmaxf(M, __ldcg(bml + ((size_t)s * GT + g) * 2));
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    for (int s = lane; s < p.splits; s += 32) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(bml + ((size_t)s * GT + g) * 2));
      const float f = (M == -INFINITY || ml.x == -INFINITY) ? 0.f : __expf(ml.x - M);
      wts[s * GT + g] = f;
      Lsum += f * ml.y;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if (lane == 0) wts[p.splits * GT + g] = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
  }
  __syncthreads();

  float racc[OPL];
#pragma unroll
  for (int i = 0; i < OPL; ++i) racc[i] = 0.f;
  for (int s0 = warp; s0 < p.splits; s0 += kU * kWarps) {
    if (s0 != warp) load_step(s0);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int s = s0 + u * kWarps;
      if (s < p.splits) {
        const float wa = wts[s * GT + gl];
#pragma unroll
        for (int i = 0; i < OPL; ++i) racc[i] += wa * va[u][i];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < OPL; i += VW) {
    if constexpr (VW == 4) {
      *reinterpret_cast<float4*>(red + warp * GT * DC + e0 + i) = make_float4(racc[i], racc[i + 1], racc[i + 2], racc[i + 3]);
    } else {
      *reinterpret_cast<float2*>(red + warp * GT * DC + e0 + i) = make_float2(racc[i], racc[i + 1]);
    }
  }
  __syncthreads();
  for (int e = tid; e < GT * DC; e += kThreads) {
    const int g = e / DC, c = c_base + e % DC;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[w * GT * DC + e];
    const int hq = h * p.G + gz * GT + g;
    p.out[((size_t)b * p.Hq + hq) * D + c] = v * wts[p.splits * GT + g];
  }
}

// Shared-memory bytes of a plan.
template <int D, int GT>
int plan_smem(int split_len, int splits, bool with_lg = true) {
  return smem_layout<D, GT>(split_len, splits, with_lg).total;
}

template <int D, int GT, bool GATED, bool PAGED, bool DENSE>
cudaError_t launch_t(const AttendParams& p0, cudaStream_t stream) {
  auto kern = attend_kernel<D, GT, GATED, PAGED, DENSE>;
  AttendParams p = p0;
  if (p.sms > 0) {
    // Re-split for whole waves: CTAs resident per SM at the largest slice, then the split count
    // in [s_lo, max_splits] whose grid fills its last wave best (the most splits when even
    // max_splits does not fill one wave).  The dense variant's count is the cache capacity.
    const int count_max = p.k_max;
    const int max_len = DENSE ? kMaxSplitLenDense : kMaxSplitLen;
    const int occ = ctas_per_sm((const void*)kern, kThreads, plan_smem<D, GT>(max_len, p.max_splits, GATED));
    const long heads = (long)p.B * p.Hkv * p.ngz;
    const long slots = (long)p.sms * occ;
    const int s_lo = (count_max + max_len - 1) / max_len;
    int best = p.max_splits;
    if (DENSE) {
      // The dense slices are long and bandwidth-bound: balance the rows per SM (CTAs a multiple
      // of the SM count) and keep the resident slots filled; one wave when one can hold them.
      // Each candidate is scored on its split count after the slice length is rounded.
      const bool one_wave = heads * s_lo <= slots;
      double best_eff = -1.0;
      for (int s = s_lo < 1 ? 1 : s_lo; s <= p.max_splits; ++s) {
        int len = (count_max + s - 1) / s;
        len = (len + 31) & ~31;
        const long ctas = heads * (long)((count_max + len - 1) / len);
        if (one_wave && ctas > slots) break;
        const long per_sm = (ctas + p.sms - 1) / p.sms;
        const double fill = (double)(ctas < slots ? ctas : slots) / (double)slots;
        const double eff = fill * (double)ctas / (double)(per_sm * p.sms);
        if (eff > best_eff + 1e-9) {
          best_eff = eff;
          best = s;
        }
      }
    } else if (heads * p.max_splits > slots) {
      double best_eff = -1.0;
      for (int s = s_lo < 1 ? 1 : s_lo; s <= p.max_splits; ++s) {
        const long ctas = heads * s;
        const long waves = (ctas + slots - 1) / slots;
        const double eff = (double)ctas / (double)(waves * slots);
        if (eff > best_eff + 1e-9) {
          best_eff = eff;
          best = s;
        }
        if (eff >= 0.9) break;
      }
    }
    int len = (count_max + best - 1) / best;
    len = (len + 31) & ~31;
    if (len < 32) len = 32;
    p.split_len = len;
    p.splits = (count_max + len - 1) / len;
  }
  p.smem_bytes = plan_smem<D, GT>(p.split_len, p.splits, GATED);
  cudaError_t e = prepare_kernel((const void*)kern, p.smem_bytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.splits, (unsigned)(p.B * p.Hkv), (unsigned)p.ngz);
  e = launch_pdl(kern, grid, dim3(kThreads), (size_t)p.smem_bytes, stream, p);
  if (e != cudaSuccess) return e;
  // Few head groups: four CTAs per group, each merging a quarter of the channels.
  const unsigned groups = (unsigned)(p.B * p.Hkv * p.ngz);
  if constexpr (GT * D / 4 >= 64) {
    if (p.sms > 0 && groups * 2 < (unsigned)p.sms) {
      auto ck = combine_kernel<D, GT, 4>;
      const int csm = combine_smem_floats<D, GT, 4>(p.splits) * 4;
      e = prepare_kernel((const void*)ck, csm);
      if (e != cudaSuccess) return e;
      return launch_pdl(ck, dim3(groups, 4), dim3(kThreads), (size_t)csm, stream, p);
    }
  }
  auto ck = combine_kernel<D, GT, 1>;
  const int csm = combine_smem_floats<D, GT, 1>(p.splits) * 4;
  e = prepare_kernel((const void*)ck, csm);
  if (e != cudaSuccess) return e;
  return launch_pdl(ck, dim3(groups), dim3(kThreads), (size_t)csm, stream, p);
}

template <int D, int GT>
cudaError_t launch_dg(const AttendParams& p, cudaStream_t stream) {
  const bool dense = (p.idx == nullptr);
  const bool gated = (p.log_g != nullptr);
  const bool paged = p.paged != 0;
  if (dense) return paged ? launch_t<D, GT, false, true, true>(p, stream) : launch_t<D, GT, false, false, true>(p, stream);
  if (gated) return paged ? launch_t<D, GT, true, true, false>(p, stream) : launch_t<D, GT, true, false, false>(p, stream);
  return paged ? launch_t<D, GT, false, true, false>(p, stream) : launch_t<D, GT, false, false, false>(p, stream);
}

template <int D>
cudaError_t launch_d(const AttendParams& p, cudaStream_t stream) {
  switch (p.gt) {
    case 4: return launch_dg<D, 4>(p, stream);
    case 2: return launch_dg<D, 2>(p, stream);
    case 1: return launch_dg<D, 1>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

void plan_attend(AttendParams& p, int count_max, bool dense) {
  p.gt = (p.G % 4 == 0) ? 4 : ((p.G % 2 == 0) ? 2 : 1);
  p.ngz = p.G / p.gt;
  const long heads = (long)p.B * p.Hkv * p.ngz;
  if (count_max < 1) count_max = 1;
  const long maxlen = dense ? kMaxSplitLenDense : kMaxSplitLen;
  long s = (kTargetCtas + heads - 1) / heads;
  if (s < 1) s = 1;
  long len = (count_max + s - 1) / s;
  len = (len + 31) & ~31L;
  if (len < kMinSplitLen) len = kMinSplitLen;
  const long cm32 = ((long)count_max + 31) & ~31L;
  if (len > cm32) len = cm32;
  if (len > maxlen) len = maxlen;
  p.split_len = (int)len;
  p.splits = (int)((count_max + len - 1) / len);
  p.max_splits = p.splits;
  if (!dense) {
    int more = (count_max + kMinSplitLen - 1) / kMinSplitLen;
    if (more > kMaxSplitsPerHead) more = kMaxSplitsPerHead;
    if (more > p.max_splits) p.max_splits = more;
  }
  int smem;
  if (p.d == 128) {
    smem = (p.gt == 4) ? plan_smem<128, 4>(p.split_len, p.splits)
                       : (p.gt == 2 ? plan_smem<128, 2>(p.split_len, p.splits) : plan_smem<128, 1>(p.split_len, p.splits));
  } else {
    smem = (p.gt == 4) ? plan_smem<64, 4>(p.split_len, p.splits)
                       : (p.gt == 2 ? plan_smem<64, 2>(p.split_len, p.splits) : plan_smem<64, 1>(p.split_len, p.splits));
  }
  p.smem_bytes = smem;
}

size_t attend_workspace_floats(const AttendParams& p) {
  return (size_t)p.B * p.Hkv * p.ngz * p.max_splits * p.gt * (p.d + 2);
}

cudaError_t launch_attend(const AttendParams& p, cudaStream_t stream) {
  if (p.d == 128) return launch_d<128>(p, stream);
  if (p.d == 64) return launch_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sas
