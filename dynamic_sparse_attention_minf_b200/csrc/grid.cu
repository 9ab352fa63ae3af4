// Row permutations of the Grid pattern (MMInference abstract: the temporal
// and spatial locality of video gives a Grid pattern, handled through a
// permutation).  A video segment of F frames x P tokens per frame is stored
// frame-major, token i = f * P + p; gathering the tokens of each in-frame
// position p into a sequence of its own (position-major order) turns the
// segment [B, H, F * P, d] into [B * P, H, F, d], where Block-Sparse
// estimation and attention run unchanged, and the output goes back the
// same way.
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

namespace {

// One row of d bf16 (d * 2 bytes) per group of d / 8 threads, 16 bytes each.
// Rows are enumerated over (head slot, batch, position, frame); `dir` = 0
// copies frame-major rows into position-major ones, 1 the other way.
__global__ void __launch_bounds__(256) grid_permute_kernel(const GridPermParams p) {
  const int tpr = p.d / 8;  // threads per row
  const long long t = (long long)blockIdx.x * 256 + threadIdx.x;
  const long long row = t / tpr;
  const int q = (int)(t % tpr);
  const long long rows = (long long)p.nh * p.B * p.N;
  if (row >= rows) return;
  const int f = (int)(row % p.F);
  long long r = row / p.F;
  const int pos = (int)(r % p.P);
  r /= p.P;
  const int b = (int)(r % p.B);
  const int hi = (int)(r / p.B);
  const int head = p.heads ? __ldg(p.heads + hi) : hi;
  if (head < 0 || head >= p.H) {
    if (q == 0 && f == 0 && pos == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 70);
    return;
  }
  const size_t frame_major = ((size_t)b * p.H + head) * p.N + (size_t)f * p.P + pos;
  const size_t pos_major = (((size_t)b * p.P + pos) * p.H + head) * p.F + f;
  const size_t src = p.dir == 0 ? frame_major : pos_major;
  const size_t dst = p.dir == 0 ? pos_major : frame_major;
  reinterpret_cast<uint4*>(p.dst + dst * p.d)[q] = __ldg(reinterpret_cast<const uint4*>(p.src + src * p.d) + q);
  if (p.lse_src && q == 0) p.lse_dst[dst] = p.lse_src[src];
}

}  // namespace

cudaError_t grid_permute_launch(const GridPermParams& p, cudaStream_t stream) {
  const long long threads = (long long)p.nh * p.B * p.N * (p.d / 8);
  if (threads == 0) return cudaSuccess;
  grid_permute_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace minf
