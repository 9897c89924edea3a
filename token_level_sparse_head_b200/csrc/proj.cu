// Projected score cache: Kproj = K M^T stored as bf16 (sm_100a).
//
// JSSA page, section 投影打分缓存与校准成本: besides the raw bf16 KV cache, a low-rank key
// cache Kproj = K M^T (M in R^{r x d}, orthonormal rows, one per KV head) is kept for token
// selection only.  Section 组件级拆解 / Figure 9: projecting each new key is the cheapest
// phase of the step.
//
// build : every cached row i < N_b of every (b, h), one thread per row, M[h] staged in shared
//         memory and read as broadcast float4s;
// append: the newest key of every (b, h), one warp per (b, h), one lane per output element.
// Both accumulate each output in fp32 in channel order c = 0..d-1 (so an appended row is
// bit-identical to the same row built), then round to bf16 (nearest even).
#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kBuildThreads = 256;

template <int D, int R>
__global__ void __launch_bounds__(kBuildThreads) build_kernel(const ProjParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ms = reinterpret_cast<float*>(smem_raw);
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const float4* Mg = reinterpret_cast<const float4*>(p.M + (size_t)h * R * D);
  for (int e = threadIdx.x; e < R * D / 4; e += kBuildThreads) reinterpret_cast<float4*>(Ms)[e] = Mg[e];
  __syncthreads();

  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && h == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    return;
  }
  const int i = blockIdx.x * p.rows_per_cta + threadIdx.x;
  if (i >= n) return;
  size_t row;
  if (p.paged) {
    const int pg = p.page_table[(size_t)b * p.max_pages + (i >> 6)];
    if (pg < 0 || pg >= p.num_pages) {
      record_error(p.err, kDevBadPage, (uint32_t)b);
      return;
    }
    row = ((size_t)pg * p.Hkv + h) * 64 + (i & 63);
  } else {
    row = (size_t)bh * p.cap + i;
  }
  // The key row is re-read (L1-resident) once per block of 16 outputs, 4 channels at a time.
  const uint2* src = reinterpret_cast<const uint2*>(p.K + row * D);
  uint32_t outw[R / 2];
  constexpr int JB = 16;
#pragma unroll
  for (int jb = 0; jb < R; jb += JB) {
    float acc[JB];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) acc[jj] = 0.f;
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const uint2 kk = src[c4];
      const float k0 = bf16lo(kk.x), k1 = bf16hi(kk.x);
      const float k2 = bf16lo(kk.y), k3 = bf16hi(kk.y);
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) {
        const float4 m = reinterpret_cast<const float4*>(Ms + (size_t)(jb + jj) * D)[c4];
        float a = acc[jj];
        a = fmaf(m.x, k0, a);
        a = fmaf(m.y, k1, a);
        a = fmaf(m.z, k2, a);
        a = fmaf(m.w, k3, a);
        acc[jj] = a;
      }
    }
#pragma unroll
    for (int jj = 0; jj < JB; jj += 2) {
      const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[jj], acc[jj + 1]);
      outw[(jb + jj) / 2] = *reinterpret_cast<const uint32_t*>(&pr);
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(p.Kproj + row * R);
#pragma unroll
  for (int v = 0; v < R / 8; ++v) dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
}

// One warp per (b, h): lane j computes outputs j, j+32.
template <int D, int R>
__global__ void __launch_bounds__(256) append_kernel(const ProjParams p) {
  __shared__ float ks[8][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 8 + warp;
  if (bh >= p.B * p.Hkv) return;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (lane == 0 && h == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    return;
  }
  if (n == 0) return;
  const int i = n - 1;
  const __nv_bfloat16* kn = p.K + (size_t)bh * D;
  for (int c = lane; c < D; c += 32) ks[warp][c] = __bfloat162float(kn[c]);
  __syncwarp();
  size_t row;
  if (p.paged) {
    const int pg = p.page_table[(size_t)b * p.max_pages + (i >> 6)];
    if (pg < 0 || pg >= p.num_pages) {
      if (lane == 0) record_error(p.err, kDevBadPage, (uint32_t)b);
      return;
    }
    row = ((size_t)pg * p.Hkv + h) * 64 + (i & 63);
  } else {
    row = (size_t)bh * p.cap + i;
  }
#pragma unroll
  for (int j = lane; j < R; j += 32) {
    const float* Mj = p.M + ((size_t)h * R + j) * D;
    float a = 0.f;
    for (int c = 0; c < D; ++c) a = fmaf(Mj[c], ks[warp][c], a);
    p.Kproj[row * R + j] = __float2bfloat16_rn(a);
  }
}

template <int D, int R>
cudaError_t launch_dr(const ProjParams& p, cudaStream_t stream) {
  if (p.append) {
    const int blocks = (p.B * p.Hkv + 7) / 8;
    append_kernel<D, R><<<blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)R * D * 4;
  auto kern = build_kernel<D, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.cap + p.rows_per_cta - 1) / p.rows_per_cta), (unsigned)(p.B * p.Hkv), 1);
  kern<<<grid, kBuildThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const ProjParams& p, cudaStream_t stream) {
  switch (p.r) {
    case 16: return launch_dr<D, 16>(p, stream);
    case 32: return launch_dr<D, 32>(p, stream);
    case 64: return launch_dr<D, 64>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_proj(const ProjParams& p0, cudaStream_t stream) {
  ProjParams p = p0;
  p.rows_per_cta = kBuildThreads;
  if (p.d == 128) return launch_d<128>(p, stream);
  if (p.d == 64) return launch_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sas
