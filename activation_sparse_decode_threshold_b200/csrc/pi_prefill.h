// pi_prefill.h -- internal interface of the dense multi-token prefill path.
#pragma once
#include <cuda_runtime.h>

#include <vector>

#include "pi_internal.h"

namespace pi {

struct PrefillState;

// What the prefill needs from a handle (weights in neuron-table order).
struct PrefillView {
    int n_layers;
    int d, F, E, top_k, act, gated, wfmt, wrow;
    int rec_bytes, wd_stride;                   // neuron record stride, W_down row stride (bytes)
    float eps;
    const ExpertDev *ex;                        // host copy [n_layers * E]
    uint8_t *const *router;                     // host copy [n_layers] device pointers
    const std::vector<std::vector<int32_t>> *perm;
    int *err;                                   // the handle's device error word
    long long wait_ns;                          // bound on every device-side wait
    int debug_flags;                            // PI_DEBUG_* testing aids
};

// Returns 0 on success, 1 unsupported, 2 CUDA error, 3 out of memory; `msg`
// describes a failure.
int prefill_run(PrefillState **state, const PrefillView &v, int l0, int l1, int T, float *resid,
                cudaStream_t stream, char *msg, int msg_len);
void prefill_invalidate(PrefillState *state, int layer);
void prefill_destroy(PrefillState *state);

}  // namespace pi
