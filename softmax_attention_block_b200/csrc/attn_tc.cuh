// Tensor-core (tcgen05) versions of the attention main loops.
#pragma once
#include "attn.cuh"

namespace path {

struct FwdTcArgs {
    const float *Sd;   // [nh, nblk, BT, BT] diagonal-block logits (bilinear term)
    const float *c;    // [nh, Lp] gate prefix or null
    float scale_log2;  // scale * log2(e)
    int L, nblk, nh;
    long long npairs;
    void *out;
    float *lse;
    int *err;          // device error word (first wait that gave up)
};

bool attn_fwd_tc_supported(Types t, int d);
cudaError_t attn_fwd_tc(const FwdArgs &f, Types t, int d, int *err, cudaStream_t st);

}  // namespace path
