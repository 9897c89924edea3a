// Gather of the selected K/V rows into contiguous buffers (sm_100a) -- the staging copy that a
// gather-based sparse attention makes and the library's own attention avoids.
//
// JSSA page, section 原理详解(二) / gather 到底贵在哪: materialising the selected entries costs
// about as much as the attention over them.  This kernel exists to measure that on the same
// hardware: followed by the dense decode over the gathered rows it computes what the
// gather-free attention computes.  CTA (b, h, slice of 128 index entries); every thread moves
// 16-byte pieces of K and V rows, consecutive threads consecutive pieces of a row.
#include "sas_device.cuh"
#include "sas_kernels.h"

namespace sas {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerCta = 128;

template <int D>
__global__ void __launch_bounds__(kThreads) gather_kernel(const GatherParams p) {
  pdl_wait();
  pdl_trigger();
  const int bh = blockIdx.x;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  int n = p.seqlens[b];
  if (n < 0 || n > p.cap) n = 0;
  const int cnt = max(0, min(min(p.kvec[b], p.k_max), n));
  if (blockIdx.y == 0 && h == 0 && threadIdx.x == 0) p.counts[b] = cnt;
  const int j0 = blockIdx.y * kRowsPerCta;
  const int j1 = min(j0 + kRowsPerCta, cnt);
  constexpr int PPR = D / 8;  // 16-byte pieces per row
  const int32_t* idx = p.idx + (size_t)bh * p.k_max;
  for (int e = j0 * PPR + threadIdx.x; e < j1 * PPR; e += kThreads) {
    const int j = e / PPR, part = e % PPR;
    int pos = idx[j];
    if (pos < 0 || pos >= n) pos = 0;  // entries outside [0, N_b) read position 0
    size_t row;
    if (p.paged) {
      int pg = p.page_table[(size_t)b * p.max_pages + (pos >> 6)];
      if (pg < 0 || pg >= p.num_pages) pg = 0;
      row = ((size_t)pg * p.Hkv + h) * 64 + (pos & 63);
    } else {
      row = (size_t)bh * p.cap + pos;
    }
    const size_t dst = ((size_t)bh * p.k_max + j) * D + part * 8;
    const uint4 kv = ldg_stream128(p.K + row * D + part * 8);
    const uint4 vv = ldg_stream128(p.V + row * D + part * 8);
    *reinterpret_cast<uint4*>(p.Kg + dst) = kv;
    *reinterpret_cast<uint4*>(p.Vg + dst) = vv;
  }
}

}  // namespace

cudaError_t launch_gather(const GatherParams& p, cudaStream_t stream) {
  const dim3 grid((unsigned)(p.B * p.Hkv), (unsigned)((p.k_max + kRowsPerCta - 1) / kRowsPerCta), 1);
  if (p.d == 128) return launch_pdl(gather_kernel<128>, grid, dim3(kThreads), 0, stream, p);
  if (p.d == 64) return launch_pdl(gather_kernel<64>, grid, dim3(kThreads), 0, stream, p);
  return cudaErrorInvalidValue;
}

}  // namespace sas
