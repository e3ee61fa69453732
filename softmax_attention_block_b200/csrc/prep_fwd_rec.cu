// Forward UT prep of one 128-position block as direct recurrences (fp32).
//
// Within block J (positions s..e, H_t = I - beta_t w_t w_t^T) the forward
// needs four things, each a product of the block's H factors:
//   Ktil_j = H_e ... H_{j+1} k_j          (keys carried to the block end)
//   Qtil_i = H_s ... H_i q_i              (queries carried back to the block start;
//                                          as a row, q_i^T H_i ... H_s)
//   P      = H_e ... H_s                  (the block product)
//   Sd_ij  = q_i^T H_i ... H_{j+1} k_j    (j <= i: the logits inside the block)
// They are the quantities the UT transform expresses in closed form
// (Paper-Notes "训练策略": I - W^T T^{-1} W, and the full-matrix form). Here
// each is the sequence of rank-one updates itself, run by one thread per
// row or column: thread j carries k_j through H_{j+1}, ..., H_e and emits
// Sd_tj = q_t . k_j after every step (the in-place key update of the
// inference paragraph, applied inside the block); thread i carries q_i
// through H_i, ..., H_s; thread c carries column c of I through H_s, ..., H_e.
// The three roles are separate CTAs of 128 threads, so that a thread's vector
// of up to 128 fp32 values stays in registers.
// Positions past the sequence end have beta = 0 and w = 0 (H = I).
#include "prep.cuh"
#include "runtime.cuh"

namespace path {

namespace {

template <int D>
struct RecCfg {
    // one role per CTA (grid z: 0 keys, 1 queries, 2 columns of P), one vector
    // of D fp32 values per thread, kept in registers
    static constexpr int NT = BT;
    static constexpr int LDS = D + 4;  // shared row stride: 16-byte rows for vector reads
};

// Dot product of row t of a shared [BT][D + 4] matrix with x. Every thread of
// the warp reads the same row: broadcast 16-byte loads.
template <int D>
__device__ __forceinline__ float row_dot(const float *sm, int t, const float (&x)[D])
{
    const float4 *p = reinterpret_cast<const float4 *>(sm + t * RecCfg<D>::LDS);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 v = p[c];
        s0 = fmaf(v.x, x[4 * c], s0);
        s1 = fmaf(v.y, x[4 * c + 1], s1);
        s2 = fmaf(v.z, x[4 * c + 2], s2);
        s3 = fmaf(v.w, x[4 * c + 3], s3);
    }
    return (s0 + s1) + (s2 + s3);
}

// x <- H_t x = x - beta_t w_t (w_t . x)
template <int D>
__device__ __forceinline__ void apply_h(float (&x)[D], const float *sW, const float *sB, int t)
{
    const float coef = sB[t] * row_dot<D>(sW, t, x);
    const float4 *p = reinterpret_cast<const float4 *>(sW + t * RecCfg<D>::LDS);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 v = p[c];
        x[4 * c] = fmaf(-coef, v.x, x[4 * c]);
        x[4 * c + 1] = fmaf(-coef, v.y, x[4 * c + 1]);
        x[4 * c + 2] = fmaf(-coef, v.z, x[4 * c + 2]);
        x[4 * c + 3] = fmaf(-coef, v.w, x[4 * c + 3]);
    }
}

template <typename T, typename TM, int D>
__global__ void __launch_bounds__(RecCfg<D>::NT)
    prep_fwd_rec_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ w,
                        const float *__restrict__ beta, int L, int nblk, TM *Qt, TM *Kt, TM *Pm,
                        float *Sd, int role0)
{
    constexpr int LDS = RecCfg<D>::LDS;
    extern __shared__ __align__(16) float sm[];
    float *sW = sm;              // [BT][D+4]
    float *sB = sW + BT * LDS;   // [BT]
    float *sQ = sB + BT;         // [BT][D+4], keys role only
    const int J = blockIdx.x, h = blockIdx.y, role = role0 + blockIdx.z, tid = threadIdx.x;
    const int Lp = nblk * BT;
    const long long row0 = (long long)h * L + (long long)J * BT;  // first row of the block in [nh, L]
    const int nvalid = min(BT, L - J * BT);
    for (int e = tid; e < BT * D; e += blockDim.x) {
        const int r = e / D, c = e % D;
        const bool ok = r < nvalid;
        sW[r * LDS + c] = ok ? to_f(w[(row0 + r) * D + c]) : 0.f;
        if (role == 0) sQ[r * LDS + c] = ok ? to_f(q[(row0 + r) * D + c]) : 0.f;
    }
    for (int r = tid; r < BT; r += blockDim.x) sB[r] = r < nvalid ? beta[row0 + r] : 0.f;
    __syncthreads();

    if (role == 0) {
        // keys: Ktil and the diagonal-block logits
        const int j = tid;
        float x[D];
#pragma unroll
        for (int c = 0; c < D; ++c) x[c] = j < nvalid ? to_f(k[(row0 + j) * D + c]) : 0.f;
        float *sd = Sd + ((long long)h * nblk + J) * BT * BT;
        sd[(long long)j * BT + j] = row_dot<D>(sQ, j, x);
        // the step index is the same for the whole warp (broadcast rows);
        // lanes with t <= j only write the zero above the diagonal
        for (int t = (j & ~31) + 1; t < BT; ++t) {
            if (t > j) {
                apply_h<D>(x, sW, sB, t);
                sd[(long long)t * BT + j] = row_dot<D>(sQ, t, x);
            } else if (t < j) {
                sd[(long long)t * BT + j] = 0.f;  // above the diagonal (never read)
            }
        }
        for (int t = 0; t < (j & ~31); ++t) sd[(long long)t * BT + j] = 0.f;
        TM *dst = Kt + ((long long)h * Lp + (long long)J * BT + j) * D;
#pragma unroll
        for (int c = 0; c < D; ++c) dst[c] = from_f<TM>(x[c]);
    } else if (role == 1) {
        // queries: Qtil_i = H_s ... H_i q_i (apply H_i first)
        const int i = tid;
        float x[D];
#pragma unroll
        for (int c = 0; c < D; ++c) x[c] = i < nvalid ? to_f(q[(row0 + i) * D + c]) : 0.f;
        for (int t = (i | 31); t >= 0; --t)
            if (t <= i) apply_h<D>(x, sW, sB, t);
        TM *dst = Qt + ((long long)h * Lp + (long long)J * BT + i) * D;
#pragma unroll
        for (int c = 0; c < D; ++c) dst[c] = from_f<TM>(x[c]);
    } else {
        // block product P = H_e ... H_s, one column per thread
        const int col = tid;
        if (col < D) {
            float x[D];
#pragma unroll
            for (int c = 0; c < D; ++c) x[c] = c == col ? 1.f : 0.f;
            for (int t = 0; t < BT; ++t) apply_h<D>(x, sW, sB, t);
            TM *dst = Pm + ((long long)h * nblk + J) * D * D;
#pragma unroll
            for (int r = 0; r < D; ++r) dst[(long long)r * D + col] = from_f<TM>(x[r]);
        }
    }
}

template <typename T, typename TM, int D>
cudaError_t run(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out, cudaStream_t st)
{
    // keys (W, beta and Q in shared memory), then queries and P columns (W, beta)
    const size_t smem_w = (BT * RecCfg<D>::LDS + BT) * sizeof(float);
    const size_t smem_k = smem_w + BT * RecCfg<D>::LDS * sizeof(float);
    auto kern = prep_fwd_rec_kernel<T, TM, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k);
    if (e != cudaSuccess) return e;
    for (int role0 = 0; role0 < 2; ++role0) {
        kern<<<dim3(Dm.nblk, Dm.nh, role0 == 0 ? 1 : 2), RecCfg<D>::NT, role0 == 0 ? smem_k : smem_w, st>>>(
            static_cast<const T *>(in.q), static_cast<const T *>(in.k), static_cast<const T *>(in.w),
            in.beta, Dm.L, Dm.nblk, static_cast<TM *>(out.Qt), static_cast<TM *>(out.Kt),
            static_cast<TM *>(out.Pm), out.Sd, role0);
        count_launches();
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int D>
cudaError_t by_types(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out, cudaStream_t st)
{
    if (Dm.dt == F32) return run<float, float, D>(Dm, in, out, st);
    return run<bf16, f16, D>(Dm, in, out, st);
}

}  // namespace

cudaError_t prep_forward_rec(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out,
                             cudaStream_t st)
{
    switch (Dm.d) {
    case 16: return by_types<16>(Dm, in, out, st);
    case 32: return by_types<32>(Dm, in, out, st);
    case 64: return by_types<64>(Dm, in, out, st);
    case 128: return by_types<128>(Dm, in, out, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace path
