// pi_prefill.cu -- dense multi-token prefill on the tensor cores.
#include <cstdio>

#include "pi_prefill.h"

namespace pi {

struct PrefillState {
    int dummy;
};

int prefill_run(PrefillState **state, const PrefillView &v, int l0, int l1, int T, float *resid,
                cudaStream_t stream, char *msg, int msg_len)
{
    (void)state; (void)v; (void)l0; (void)l1; (void)T; (void)resid; (void)stream;
    snprintf(msg, msg_len, "dense prefill is not available in this build");
    return 1;
}

void prefill_invalidate(PrefillState *, int) {}

void prefill_destroy(PrefillState *state) { delete state; }

}  // namespace pi
