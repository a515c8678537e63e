// qstage.cu — the query of a decode step taken from pinned host memory.
//
// When q is in pinned host memory, the step first copies it across the host
// link into the workspace with this kernel, so the scan's and the finishing
// kernel's many reads of q hit HBM, not the link.  Launched as a programmatic
// dependent of the previous kernel in the stream: every thread loads its
// 16-byte pieces before waiting on that kernel (no device kernel writes host
// q), so the link's latency overlaps the previous step's finishing kernel;
// the stores come after the wait, because that kernel may still be reading
// the staged copy.  No early release of the next kernel: the finishing
// kernel reads q before its own wait, so the kernels after this one start
// only once it has exited.  One CTA of 1024 threads per 64 KB.
#include "jfa_internal.cuh"

namespace jfa {

constexpr int kQsThreads = 1024;
constexpr int kQsPer = 4;  // 16-byte pieces per thread

__global__ void __launch_bounds__(kQsThreads) q_stage_kernel(const uint4* __restrict__ src,
                                                             uint4* __restrict__ dst, int n16) {
  const int base = blockIdx.x * kQsThreads * kQsPer + threadIdx.x;
  uint4 v[kQsPer];
#pragma unroll
  for (int u = 0; u < kQsPer; ++u) {
    const int i = base + u * kQsThreads;
    v[u] = i < n16 ? src[i] : make_uint4(0u, 0u, 0u, 0u);
  }
  pdl_wait();
#pragma unroll
  for (int u = 0; u < kQsPer; ++u) {
    const int i = base + u * kQsThreads;
    if (i < n16) dst[i] = v[u];
  }
}

int stage_query(const jfa_geom& g, const uint16_t** q, uint8_t* ws, const jfa_workspace_layout& L,
                cudaStream_t st) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, *q) != cudaSuccess) {
    cudaGetLastError();
    return JFA_ERR_INVALID_ARG;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return JFA_OK;
  if (a.type != cudaMemoryTypeHost) return JFA_ERR_INVALID_ARG;  // pageable host memory
  const size_t bytes = (size_t)g.batch * g.num_heads * kD * sizeof(uint16_t);
  const int n16 = (int)(bytes / 16);
  uint16_t* dst = reinterpret_cast<uint16_t*>(ws + L.off_qstage);
  const int grid = (n16 + kQsThreads * kQsPer - 1) / (kQsThreads * kQsPer);
  if (launch_pdl(q_stage_kernel, dim3(grid), dim3(kQsThreads), 0, st,
                 reinterpret_cast<const uint4*>(*q), reinterpret_cast<uint4*>(dst), n16) != cudaSuccess)
    return JFA_ERR_CUDA;
  *q = dst;
  return JFA_OK;
}

}  // namespace jfa
