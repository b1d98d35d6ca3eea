// Row gather for the halo exchange of a spatial domain decomposition: the
// rows of a row-major device array picked by an index list, packed
// contiguously (a send buffer), in 16-byte vectors.  One GPU reaches systems
// of about 10^5 atoms ("E2Former-V2：突破等变图神经网络计算瓶颈的创新架构"
// §3.2); past that, a spatial decomposition gives each rank its own atoms,
// which it couples, and it receives the h' and k rows of the neighbours it
// does not own, once per step.
#include "egat_host.h"

namespace egat {
namespace {

__global__ void gather_rows_kernel(const uint4* __restrict__ src, long long n_src,
                                   const int32_t* __restrict__ idx, long long count, int vec,
                                   uint4* __restrict__ dst) {
  const long long total = count * vec;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long r = t / vec;
    const int v = int(t - r * vec);
    const long long j = idx[r];
    dst[t] = (j >= 0 && j < n_src) ? src[j * vec + v] : make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

int launch_gather_rows(const void* d_src, long long n_src, long long row_bytes, const int32_t* d_idx,
                       long long count, void* d_dst, cudaStream_t st) {
  if (count == 0) return EGAT_OK;
  const int vec = int(row_bytes / 16);
  const long long total = count * vec;
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  gather_rows_kernel<<<unsigned(blocks), 256, 0, st>>>(static_cast<const uint4*>(d_src), n_src, d_idx,
                                                       count, vec, static_cast<uint4*>(d_dst));
  return cudaGetLastError() == cudaSuccess ? EGAT_OK : EGAT_ERR_CUDA;
}

}  // namespace egat
