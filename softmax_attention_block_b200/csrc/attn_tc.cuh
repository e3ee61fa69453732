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
    uint64_t limit_ns; // bound on every wait of the kernel
    int withhold;      // test hook: the last query tile's producer skips one key/value load
};

struct BwdTcArgs {
    const float *Sd, *c, *lse_p, *delta;  // lse_p, delta, c: [nh, Lp]
    float scale;
    int L, nblk, nh;
    long long npairs;
    float *dQt, *dKt, *dPm, *dSd;  // dQt, dPm accumulated (zeroed by the caller)
    void *dv;
    float *rowsum, *colsum;        // rowsum accumulated (zeroed by the caller)
    int *err;
};

bool attn_bwd_tc_supported(Types t, int d);
// lse_p: [nh, Lp] scratch; dout_bf16: [nh, L, d] scratch (used when dout is fp32).
// attn_bwd_tc_prepare (per-query terms, bf16 dout) runs first on the same stream.
cudaError_t attn_bwd_tc_prepare(const BwdArgs &b, Types t, int d, float *lse_p, void *dout_bf16,
                                cudaStream_t st);
cudaError_t attn_bwd_tc(const BwdArgs &b, Types t, float *lse_p, void *dout_bf16, int *err,
                        cudaStream_t st);
// Head dim 128 (attn_bwd128_tc.cu): the same contract, 64-query sub-tiles.
bool attn_bwd128_tc_supported(Types t, int d);
cudaError_t attn_bwd128_tc(const BwdArgs &b, Types t, float *lse_p, void *dout_bf16, int *err,
                           cudaStream_t st);

bool attn_fwd_tc_supported(Types t, int d);
// Key-side transport chain (fp16 tensors, d in {64, 128}).
cudaError_t chain_tc(const ChainArgs &c, int d, int *err, cudaStream_t st);
// fp16 copy of n bf16 elements (n % 8 == 0, 16-byte aligned buffers)
cudaError_t convert_to_f16(const void *src, void *dst, long long n, cudaStream_t st);
cudaError_t attn_fwd_tc(const FwdArgs &f, Types t, int d, int *err, cudaStream_t st);

}  // namespace path
