// pivot.cu -- online dynamic pivot detection on the per-layer statistics.
//
// StructKV (gist.science 2604.06746) section 2.B: the attention entropy,
// sparsity and variance of each layer are watched as the prompt goes through
// the model, and the layer where the entropy falls sharply while the
// sparsity rises is the pivot, where the structural propagation happens.
// The page gives neither the per-layer statistic nor a threshold; the rule
// here: head-mean entropy E_l and top-1% mass S_l (float64, heads in order),
// pivot = first layer l in [max(2, l_min), l_max] with
// E_{l-1} - E_l >= tau * E_{l-1} and S_l > S_{l-1}, else l_max.
//
// The state lives in device memory and one thread folds in each layer, so a
// layer loop (or a CUDA graph of it) needs no host synchronisation to decide.
// The arithmetic is IEEE float64 with explicit round-to-nearest operations,
// so the decision is reproducible bit for bit by any float64 implementation
// of the same rule that sums the heads in the same order.
#include "common.cuh"

namespace kvc {
namespace {

__global__ void __launch_bounds__(32) pivot_update_kernel(const float* __restrict__ stats, int rows, int layer,
                                                          double tau, int l_min, int l_max, kvc_pivot_state* st,
                                                          int32_t* err) {
  pdl_wait();  // this layer's statistics come from the previous kernel
  if (threadIdx.x != 0) return;
  if (st->layers_seen != layer - 1) {
    set_dev_err(err, KVC_DEV_ERR_ORDER);
    return;
  }
  double E = 0.0, S = 0.0;
  for (int g = 0; g < rows; ++g) {
    E = __dadd_rn(E, (double)stats[(int64_t)g * 3 + 0]);
    S = __dadd_rn(S, (double)stats[(int64_t)g * 3 + 1]);
  }
  E = __ddiv_rn(E, (double)rows);
  S = __ddiv_rn(S, (double)rows);
  if (st->pivot == 0 && layer <= l_max) {
    const bool fires = layer >= 2 && layer >= l_min &&
                       __dsub_rn(st->prev_entropy, E) >= __dmul_rn(tau, st->prev_entropy) && S > st->prev_sparsity;
    if (fires || layer == l_max) st->pivot = layer;
  }
  st->prev_entropy = E;
  st->prev_sparsity = S;
  st->layers_seen = layer;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_pivot_update(const float* stats, int32_t rows, int32_t layer, double tau, int32_t l_min,
                                       int32_t l_max, kvc_pivot_state* state, int32_t* dev_err, void* stream) {
  clear_error();
  KVC_CHECK_ARG(stats != nullptr && state != nullptr, "stats and state must be non-NULL");
  KVC_CHECK_ARG(rows >= 1 && rows <= 65535, "rows out of range");
  KVC_CHECK_ARG(layer >= 1, "layer must be >= 1");
  KVC_CHECK_ARG(tau >= 0.0, "tau must be >= 0");
  KVC_CHECK_ARG(l_min >= 1 && l_max >= l_min, "need 1 <= l_min <= l_max");
  KVC_CHECK_ARG(aligned(state, 8), "state must be 8-byte aligned");
  const Launch l(dim3(1), dim3(32), 0, (cudaStream_t)stream);
  KVC_CUDA_TRY(l.run(pivot_update_kernel, stats, (int)rows, (int)layer, tau, (int)l_min, (int)l_max, state,
                     dev_err));
  count_launch();
  return KVC_OK;
}
