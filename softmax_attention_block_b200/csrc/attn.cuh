// Attention main-loop kernels (transport chain, forward, backward) and the
// forget-gate scans.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace path {

struct ChainArgs {
    const void *Kt;  // [nh, Lp, d] boundary-adjusted keys
    const void *Pm;  // [nh, nblk, d, d] block products
    void *Khat;      // [nh, npairs, BT, d]; pair (I, J), J < I, at I(I-1)/2 + J
    int nblk, nh;
};

struct FwdArgs {
    const void *Qt, *Khat, *v;
    const void *vh;   // fp16 copy of v (tensor-core path) or null
    const float *Sd;  // [nh, nblk, BT, BT]
    const float *c;   // [nh, Lp] gate prefix or null
    float scale;
    int L, nblk, nh;
    void *out;
    float *lse;
};

struct BwdArgs {
    const void *Qt, *Khat, *v, *Pm;
    const float *Sd, *c;
    float scale;
    int L, nblk, nh;
    const void *out, *dout;
    const float *lse;
    float *delta;    // [nh, Lp]
    float *dQt;      // [nh, Lp, d]
    float *dKt;      // [nh, Lp, d]
    float *dPm;      // [nh, nblk, d, d], zeroed by the caller (accumulated)
    float *dSd;      // [nh, nblk, BT, BT]
    void *dv;        // [nh, L, d]
    float *rowsum;   // [nh, Lp] or null
    float *colsum;   // [nh, Lp] or null
};

cudaError_t chain_simt(const ChainArgs &c, Types t, int d, cudaStream_t st);
cudaError_t attn_fwd_simt(const FwdArgs &a, Types t, int d, cudaStream_t st);
cudaError_t attn_bwd_simt(const BwdArgs &a, Types t, int d, cudaStream_t st);
// delta_i = dO_i . O_i into a.delta ([nh, Lp], zero past L)
cudaError_t compute_delta(const BwdArgs &a, Types t, int d, cudaStream_t st);
cudaError_t gate_prefix(const float *logf, float *c, int L, int Lp, int nh, cudaStream_t st);
cudaError_t gate_grad(const float *rowsum, const float *colsum, float *dlogf, int L, int Lp, int nh,
                      cudaStream_t st);

struct DecodeArgs {
    const void *q, *k_new, *v_new, *w;  // [nh, d]
    const float *beta;                  // [nh]
    float scale;
    int nh, n, capacity;
    void *k_cache, *v_cache;            // [nh, capacity, d]
    void *out;                          // [nh, d]
    float *partial;                     // [nh, nchunk, d + 2]
    // forget gate (both null without it): log f_t per head [nh], and each
    // cached key's logit bias c_t - c_j [nh, capacity], carried in place
    const float *log_f = nullptr;
    float *g_cache = nullptr;
};

constexpr int DECODE_CHUNK = 1024;  // cached rows per CTA

cudaError_t decode_step(const DecodeArgs &a, int dt, int d, cudaStream_t st);

// The decode cache a prefill of positions 0..L-1 leaves, from the forward's
// transported keys and block products.
struct CacheArgs {
    const void *Kt;    // [nh, Lp, d] boundary-adjusted keys (mid type)
    const void *Khat;  // [nh, npairs, BT, d] transported key tiles (mid type)
    const void *Pm;    // [nh, nblk, d, d] block products (mid type)
    const void *v;     // [nh, L, d] (input type)
    const float *c;    // [nh, Lp] gate prefix, or null
    int L, nblk, nh, capacity;
    void *k_cache, *v_cache;  // [nh, capacity, d] (input type), rows 0..L-1 written
    float *g_cache;           // [nh, capacity], rows 0..L-1 written; null without the gate
};

cudaError_t prefill_cache(const CacheArgs &a, Types t, int d, cudaStream_t st);

// Allocation-free decode: fixed device scratch of NOALLOC_SCRATCH_FLOATS.
constexpr long long NOALLOC_SCRATCH_FLOATS = 1LL << 20;
// Smallest chunk (rows per CTA) whose partials fit the fixed scratch; 0 if none.
int noalloc_chunk_rows(int nh, int n, int d);
cudaError_t noalloc_scratch(float **ptr);
cudaError_t decode_step_noalloc(const DecodeArgs &a, int dt, int d, int chunk, cudaStream_t st);

}  // namespace path
