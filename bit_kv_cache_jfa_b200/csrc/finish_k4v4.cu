// finish_k4v4.cu — the finishing kernel for 4-bit keys and 4-bit values.
#include "finish_impl.cuh"

namespace jfa {

int launch_finish_k4v4(const FinishParams& fp, int G, int n_seg, int nq_max, bool select,
                        cudaStream_t st) {
  return select ? launch_finish_g<true, 4, 4>(fp, G, n_seg, nq_max, st)
                : launch_finish_g<false, 4, 4>(fp, G, n_seg, nq_max, st);
}

}  // namespace jfa
