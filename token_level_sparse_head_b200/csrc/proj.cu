// Projected score cache: Kproj = K M^T stored as bf16, or as FP8 E4M3 codes of
// (K M^T) / kproj_scale[h] (sm_100a).
//
// JSSA page, section 投影打分缓存与校准成本: besides the raw bf16 KV cache, a low-rank key
// cache Kproj = K M^T (M in R^{r x d}, orthonormal rows, one per KV head) is kept for token
// selection only.  Section 组件级拆解 / Figure 9: projecting each new key is the cheapest
// phase of the step.
//
// build : every cached row i < N_b of every (b, h), one thread per row, M[h] staged in shared
//         memory and read as broadcast float4s;
// append: the newest key of every (b, h), one CTA per (b, h), 8 threads per output element.
// Both use one summation order for each output: 8 partial sums over consecutive blocks of d/8
// channels (fp32, in channel order), combined as ((p0+p1)+(p2+p3))+((p4+p5)+(p6+p7)), then
// rounded to bf16 (nearest even) or divided by the head's scale and rounded to E4M3 (nearest
// even, saturating at +-448); so an appended row is bit-identical to the same row built.
#include <cuda_fp8.h>

#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kBuildThreads = 256;

// Two FP8 E4M3 codes (x in the low byte) of a / s and b / s, nearest even, saturating.
__device__ __forceinline__ uint32_t fp8x2(float a, float b, float s) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a, s), __fdiv_rn(b, s)), __NV_SATFINITE, __NV_E4M3);
}

template <int D, int R, bool FP8>
__global__ void __launch_bounds__(kBuildThreads) build_kernel(const ProjParams p) {
  pdl_wait();
  pdl_trigger();
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
  // The key row is re-read (L1-resident) for each block of outputs, 4 channels at a time.
  const uint2* src = reinterpret_cast<const uint2*>(p.K + row * D);
  constexpr int BLK = D / 8;  // channels per partial sum
  constexpr int JB = 4;       // outputs per pass
  uint32_t outw[FP8 ? R / 4 : R / 2];
  const float scale = FP8 ? p.kproj_scale[h] : 1.f;
#pragma unroll
  for (int jb = 0; jb < R; jb += JB) {
    float part[JB][8];
#pragma unroll
    for (int blk = 0; blk < 8; ++blk) {
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) part[jj][blk] = 0.f;
#pragma unroll
      for (int c4 = blk * BLK / 4; c4 < (blk + 1) * BLK / 4; ++c4) {
        const uint2 kk = src[c4];
        const float k0 = bf16lo(kk.x), k1 = bf16hi(kk.x);
        const float k2 = bf16lo(kk.y), k3 = bf16hi(kk.y);
#pragma unroll
        for (int jj = 0; jj < JB; ++jj) {
          const float4 m = reinterpret_cast<const float4*>(Ms + (size_t)(jb + jj) * D)[c4];
          float a = part[jj][blk];
          a = fmaf(m.x, k0, a);
          a = fmaf(m.y, k1, a);
          a = fmaf(m.z, k2, a);
          a = fmaf(m.w, k3, a);
          part[jj][blk] = a;
        }
      }
    }
    float acc[JB];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
      const float* q = part[jj];
      acc[jj] = ((q[0] + q[1]) + (q[2] + q[3])) + ((q[4] + q[5]) + (q[6] + q[7]));
    }
    if constexpr (FP8) {
      outw[jb / 4] = fp8x2(acc[0], acc[1], scale) | (fp8x2(acc[2], acc[3], scale) << 16);
    } else {
#pragma unroll
      for (int jj = 0; jj < JB; jj += 2) {
        const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[jj], acc[jj + 1]);
        outw[(jb + jj) / 2] = *reinterpret_cast<const uint32_t*>(&pr);
      }
    }
  }
  constexpr int ROW_BYTES = FP8 ? R : 2 * R;
  uint4* dst = reinterpret_cast<uint4*>(static_cast<unsigned char*>(p.Kproj) + row * ROW_BYTES);
#pragma unroll
  for (int v = 0; v < ROW_BYTES / 16; ++v)
    dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
}

// One CTA per (b, h); thread t computes the partial of output j = t / 8 (+32 per pass) over
// channel block t % 8, and the 8 partials meet in a butterfly.
template <int D, int R, bool FP8>
__global__ void __launch_bounds__(256) append_kernel(const ProjParams p) {
  pdl_wait();
  pdl_trigger();
  const int bh = blockIdx.x;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const int n = p.seqlens[b];
  if (n < 0 || n > p.cap) {
    if (threadIdx.x == 0 && h == 0) record_error(p.err, kDevBadSeqlen, (uint32_t)b);
    return;
  }
  if (n == 0) return;
  const int i = n - 1;
  size_t row;
  if (p.paged) {
    const int pg = p.page_table[(size_t)b * p.max_pages + (i >> 6)];
    if (pg < 0 || pg >= p.num_pages) {
      if (threadIdx.x == 0) record_error(p.err, kDevBadPage, (uint32_t)b);
      return;
    }
    row = ((size_t)pg * p.Hkv + h) * 64 + (i & 63);
  } else {
    row = (size_t)bh * p.cap + i;
  }
  constexpr int BLK = D / 8;
  const int part = threadIdx.x & 7;
  float kf[BLK];
  {
    const uint32_t* kn = reinterpret_cast<const uint32_t*>(p.K + (size_t)bh * D + part * BLK);
#pragma unroll
    for (int e = 0; e < BLK / 2; ++e) {
      const uint32_t w = kn[e];
      kf[2 * e] = bf16lo(w);
      kf[2 * e + 1] = bf16hi(w);
    }
  }
#pragma unroll
  for (int pass = 0; pass < (R + 31) / 32; ++pass) {
    const int j = threadIdx.x / 8 + pass * 32;
    if (j < R) {
      const float4* Mj = reinterpret_cast<const float4*>(p.M + ((size_t)h * R + j) * D + part * BLK);
      float4 m[BLK / 4];
#pragma unroll
      for (int e = 0; e < BLK / 4; ++e) m[e] = Mj[e];
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < BLK / 4; ++e) {
        a = fmaf(m[e].x, kf[4 * e + 0], a);
        a = fmaf(m[e].y, kf[4 * e + 1], a);
        a = fmaf(m[e].z, kf[4 * e + 2], a);
        a = fmaf(m[e].w, kf[4 * e + 3], a);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      if (part == 0) {
        if constexpr (FP8) {
          static_cast<unsigned char*>(p.Kproj)[row * R + j] =
              (unsigned char)__nv_cvt_float_to_fp8(__fdiv_rn(a, p.kproj_scale[h]), __NV_SATFINITE, __NV_E4M3);
        } else {
          static_cast<__nv_bfloat16*>(p.Kproj)[row * R + j] = __float2bfloat16_rn(a);
        }
      }
    }
  }
}

template <int D, int R, bool FP8>
cudaError_t launch_drf(const ProjParams& p, cudaStream_t stream) {
  if (p.append) {
    return launch_pdl(append_kernel<D, R, FP8>, dim3((unsigned)(p.B * p.Hkv)), dim3(256), 0, stream, p);
  }
  const size_t smem = (size_t)R * D * 4;
  auto kern = build_kernel<D, R, FP8>;
  cudaError_t e = prepare_kernel((const void*)kern, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.cap + p.rows_per_cta - 1) / p.rows_per_cta), (unsigned)(p.B * p.Hkv), 1);
  return launch_pdl(kern, grid, dim3(kBuildThreads), smem, stream, p);
}

template <int D, int R>
cudaError_t launch_dr(const ProjParams& p, cudaStream_t stream) {
  return p.fp8 ? launch_drf<D, R, true>(p, stream) : launch_drf<D, R, false>(p, stream);
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
