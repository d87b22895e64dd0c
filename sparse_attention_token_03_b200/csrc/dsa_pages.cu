// Paged key caches for the chunked prefill paths: one pass gathers the
// sequence's first T_k keys from the page pool into a contiguous [T_k][128]
// bf16 matrix in the workspace, which the dense and pruned prefill kernels
// then stream with TMA tiles and gather by key id as usual.  The pass moves
// 2 x 256 bytes per key, against the O(T_q x T_k) scoring that follows.
//
//   page_gather_kernel   16 threads per key, one 16-byte load and store each;
//                        a block-table entry outside [0, n_pages) zero-fills
//                        the key and sets the overflow status bit
//   status_or_kernel     folds the gather's status word into the status word
//                        of the prefill call that ran after it
#include <algorithm>

#include "dsa_kernels.cuh"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

__global__ void page_gather_kernel(const PageGatherParams p) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t n = p.T_k * 16;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < n; g += stride) {
    const int64_t key = g >> 4;
    const int part = static_cast<int>(g & 15);
    const int32_t page = __ldg(p.block_table + key / p.page_size);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (page >= 0 && page < p.n_pages) {
      const uint16_t* src = p.k_pages + (static_cast<int64_t>(page) * p.page_size + key % p.page_size) * kD;
      v = __ldg(reinterpret_cast<const uint4*>(src) + part);
    } else if (part == 0) {
      atomicOr(p.status, kErrOverflow);
    }
    reinterpret_cast<uint4*>(p.k_out + key * kD)[part] = v;
  }
}

__global__ void status_or_kernel(const uint32_t* src, uint32_t* dst) {
  const uint32_t s = *src;
  if (s) atomicOr(dst, s);
}

}  // namespace

cudaError_t launch_page_gather(const PageGatherParams& p, int sms, cudaStream_t st) {
  if (p.T_k <= 0) return cudaSuccess;
  const int64_t threads = p.T_k * 16;
  const int grid = static_cast<int>(std::min<int64_t>((threads + 255) / 256, static_cast<int64_t>(sms) * 16));
  page_gather_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_status_or(const uint32_t* src, uint32_t* dst, cudaStream_t st) {
  status_or_kernel<<<1, 1, 0, st>>>(src, dst);
  return cudaGetLastError();
}

}  // namespace dsa
