// finish_k3v2.cu — the finishing kernel for 3-bit keys and 2-bit values.
#include "finish_impl.cuh"

namespace jfa {

int launch_finish_k3v2(const FinishParams& fp, int G, int n_seg, int nq_max, bool select,
                        cudaStream_t st) {
  return select ? launch_finish_g<true, 3, 2>(fp, G, n_seg, nq_max, st)
                : launch_finish_g<false, 3, 2>(fp, G, n_seg, nq_max, st);
}

}  // namespace jfa
