// Per-block UT transform / boundary adjustment. bf16 inputs at head dim 64: the
// tcgen05 kernels (prep_fwd_ut.cu, prep_bwd_ut.cu); at head dim 128 the forward
// on tcgen05 (prep_fwd_ut128.cu). Otherwise: the closed form by batched products
// (prep.cu; on the tensor cores for bf16 inputs), or for fp32 inputs the forward
// by recurrences in fp32 (prep_fwd_rec.cu).
#pragma once
#include "common.cuh"

namespace path {

struct PrepDims {
    int nh, L, d, nblk;
    int dt;   // element type of q, k, w
    int odt;  // element type of dq, dk, dw
};

struct PrepInputs {
    const void *q, *k, *w;  // [nh, L, d]
    const float *beta;      // [nh, L]
};

struct PrepOutputs {
    void *Qt, *Kt;  // [nh, Lp, d] boundary-adjusted queries / keys (type tdt)
    void *Pm;       // [nh, nblk, d, d] block products (type tdt)
    float *Sd;      // [nh, nblk, BT, BT] diagonal-block bilinear logits (lower part)
    int tdt;
};

struct PrepGrads {
    const float *dQt, *dKt;  // [nh, Lp, d]
    const float *dPm;        // [nh, nblk, d, d]
    const float *dSd;        // [nh, nblk, BT, BT], zero above the diagonal
    void *dq, *dk, *dw;      // [nh, L, d] (type dt)
    float *dbeta;            // [nh, L]
};

struct PrepScratch {
    float *G = nullptr, *A = nullptr, *Tinv = nullptr, *X = nullptr, *N = nullptr, *U = nullptr,
          *M = nullptr, *What = nullptr;
    float *dM = nullptr, *dU = nullptr, *dN = nullptr, *dX = nullptr, *tmp = nullptr,
          *dA = nullptr, *dG = nullptr, *dWhat = nullptr, *dWacc = nullptr;
    int *err = nullptr;  // device error word of the call
};

void carve_prep_scratch(Carver &c, const PrepDims &D, bool backward, PrepScratch &s);
size_t prep_scratch_bytes(const PrepDims &D, bool backward);
// Qtil, Ktil, P, Sd of every 128-block, computed by per-row recurrences in fp32.
cudaError_t prep_forward_rec(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                             cudaStream_t st);
// The same outputs for head dim 64 and bf16 inputs on tcgen05 (tensor memory),
// with (I + A)^{-1} as a product of block-diagonal and nilpotent factors
// (prep_fwd_ut.cu). q, k, w 16-byte aligned. err: device error word.
bool prep_forward_ut_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_forward_ut(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                            int *err, cudaStream_t st);
// Per-block quantities of the head-dim-128 UT kernels that the forward leaves for the
// adjoint (fp16, row-major; blk = head * nblk + block, h = half):
//   What [blk][h][64][128], U, X, M [blk][h][64][64], Kta, Qtb [blk][64][128]
//   (Ktil_a, Qtil_b), Pa, Pb [blk][128][128] (P_a, P_b); and the adjoint's own
//   dP [blk][h][128][128] (the halves' dP).
struct Ut128Save {
    f16 *What = nullptr, *U = nullptr, *X = nullptr, *M = nullptr, *Kta = nullptr,
        *Qtb = nullptr, *Pa = nullptr, *Pb = nullptr, *dP = nullptr;
};
void carve_ut128_save(Carver &c, const PrepDims &D, Ut128Save &s);
// The same at head dim 128 (prep_fwd_ut128.cu; outputs fp16). q, k, w 16-byte aligned.
// save: NULL, or the area the adjoint reads (prep_backward_ut128).
bool prep_forward_ut128_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_forward_ut128(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                               const Ut128Save *save, int *err, cudaStream_t st);
// Adjoint of prep_forward_ut128 from what it saved: the composition adjoint (one
// kernel per block) and the per-half UT adjoint (one kernel per half block).
// dQt and dKt are overwritten. `saved`: a device word the caller sets to bytes
// UT128_SAVED_BYTE when the save area holds the forward's values; otherwise the
// kernels record ERR_UT128_NOT_SAVED in *err and write no gradient.
constexpr int UT128_SAVED_WORD = 1;       // index in the workspace's error words
constexpr int UT128_SAVED_BYTE = 0x5A;    // memset byte of a valid save
constexpr int ERR_UT128_NOT_SAVED = 30;
cudaError_t prep_backward_ut128(const PrepDims &D, const PrepInputs &in, const PrepGrads &g,
                                const Ut128Save &save, const int *saved, int *err, cudaStream_t st);
// Adjoint of prep_forward_ut (one tcgen05 kernel per block: recomputes the halves'
// transforms, composition adjoint, per-half UT adjoint). dQt and dKt are overwritten.
bool prep_backward_ut_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_backward_ut(const PrepDims &D, const PrepInputs &in, const PrepGrads &g, int *err,
                             cudaStream_t st);
// The same outputs from the closed form by batched products (bf16 inputs at head
// dims other than 64; TF32 tensor cores), through the forward part of `s`.
cudaError_t prep_forward_gemm(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                              const PrepScratch &s, cudaStream_t st);
cudaError_t prep_backward(const PrepDims &D, const PrepInputs &in, const PrepScratch &s,
                          const PrepGrads &gr, cudaStream_t st);
cudaError_t scale_rows(const float *in, float *out, const float *beta, int L, int nblk, int batch,
                       cudaStream_t st);

}  // namespace path
