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
// Per-block quantities of the tcgen05 UT kernels (head dims 64 and 128) that the
// forward leaves for the adjoint in a backward-sized workspace (fp16, row-major;
// blk = head * nblk + block, h = half):
//   What [blk][h][64][d], U, X, M [blk][h][64][64] (M holds -lower(Q W^T)), Kta, Qtb [blk][64][d]
//   (Ktil_a, Qtil_b), Pa, Pb [blk][d][d] (P_a, P_b); at d = 128 also the
//   adjoint's own dP [blk][h][128][128] (the halves' dP).
struct UtSave {
    f16 *What = nullptr, *U = nullptr, *X = nullptr, *M = nullptr, *Kta = nullptr,
        *Qtb = nullptr, *Pa = nullptr, *Pb = nullptr, *dP = nullptr;
};
void carve_ut_save(Carver &c, const PrepDims &D, UtSave &s);
// A device word of the workspace tells the adjoint whether the save area holds the
// forward's values (bytes UT_SAVED_BYTE); without them the adjoint kernels record
// ERR_UT_NOT_SAVED in the error word and write no gradient.
constexpr int UT_SAVED_WORD = 1;       // index in the workspace's error words
constexpr int UT_SAVED_BYTE = 0x5A;    // memset byte of a valid save
constexpr int ERR_UT_NOT_SAVED = 30;
// The same outputs for head dim 64 and bf16 inputs on tcgen05 (tensor memory),
// with (I + A)^{-1} as a product of block-diagonal and nilpotent factors
// (prep_fwd_ut.cu). q, k, w 16-byte aligned. err: device error word. save: NULL,
// or the area the adjoint reads (prep_backward_ut).
bool prep_forward_ut_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_forward_ut(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                            const UtSave *save, int *err, cudaStream_t st);
// The same at head dim 128 (prep_fwd_ut128.cu; outputs fp16). q, k, w 16-byte aligned.
// save: NULL, or the area the adjoint reads (prep_backward_ut128).
bool prep_forward_ut128_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_forward_ut128(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                               const UtSave *save, int *err, cudaStream_t st);
// Adjoint of prep_forward_ut128 from what it saved: the composition adjoint (one
// kernel per block) and the per-half UT adjoint (one kernel per half block).
// dQt and dKt are overwritten. saved: the workspace's save word (UT_SAVED_WORD).
cudaError_t prep_backward_ut128(const PrepDims &D, const PrepInputs &in, const PrepGrads &g,
                                const UtSave &save, const int *saved, int *err, cudaStream_t st);
// Adjoint of prep_forward_ut from what it saved: one kernel per half block forms
// the half's adjoints from the block's (composition adjoint) and applies the UT
// adjoint. dQt and dKt are read only. saved: the workspace's save word
// (UT_SAVED_WORD).
bool prep_backward_ut_supported(const PrepDims &D, const PrepInputs &in);
cudaError_t prep_backward_ut(const PrepDims &D, const PrepInputs &in, const PrepGrads &g,
                             const UtSave &save, const int *saved, int *err, cudaStream_t st);
// The same outputs from the closed form by batched products (bf16 inputs at head
// dims other than 64; TF32 tensor cores), through the forward part of `s`.
cudaError_t prep_forward_gemm(const PrepDims &D, const PrepInputs &in, const PrepOutputs &out,
                              const PrepScratch &s, cudaStream_t st);
cudaError_t prep_backward(const PrepDims &D, const PrepInputs &in, const PrepScratch &s,
                          const PrepGrads &gr, cudaStream_t st);
cudaError_t scale_rows(const float *in, float *out, const float *beta, int L, int nblk, int batch,
                       cudaStream_t st);

}  // namespace path
