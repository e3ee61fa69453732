// Key-side block transport on tensor cores: for each key block J and every
// later block I, the keys of block J as the in-place-updated key cache holds
// them when block I starts,
//   Khat_{I,J} = Ktil_J P_{J+1}^T ... P_{I-1}^T   (row form),
// i.e. the right-to-left scan of gist.science section 3 carried on the key
// side so that each product is formed once and stored for the forward and
// backward passes. One CTA per (J, head) walks its chain: X <- X P_I^T is one
// 128 x d x d MMA (fp16 operands, fp32 in TMEM); the fp32 result is rounded to
// fp16 into the next operand buffer and stored to its pair tile by TMA.
#include "attn.cuh"
#include "attn_tc.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

template <int D>
struct ChainCfg {
    static constexpr int TILE = 128 * D * 2;
    static constexpr int PB = D * D * 2;
    static constexpr int X_OFF = 0;              // X[2]
    static constexpr int P_OFF = 2 * TILE;       // Pb[2]
    static constexpr int BAR_OFF = P_OFF + 2 * PB;
    static constexpr int SMEM = BAR_OFF + 128 + 1024;
    static constexpr uint32_t TMEM_COLS = D;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
__global__ void __launch_bounds__(128)
    chain_tc_kernel(const __grid_constant__ CUtensorMap mKt, const __grid_constant__ CUtensorMap mP,
                    const __grid_constant__ CUtensorMap mKh, int nblk, long long npairs, int *err)
{
    using C = ChainCfg<D>;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    uint8_t *X[2] = {sm + C::X_OFF, sm + C::X_OFF + C::TILE};
    uint8_t *Pb[2] = {sm + C::P_OFF, sm + C::P_OFF + C::PB};
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BAR_OFF);
    uint64_t *x_full = bars, *p_full = bars + 1, *mma_done = bars + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
    const int J = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid / 32;
    const int Lp = nblk * BT;
    const int last = nblk - 1;  // chain produces Khat_{I,J} for I = J+1 .. last
    auto pair_row = [&](int I) { return (int)((h * npairs + (long long)I * (I - 1) / 2 + J) * BT); };

    if (tid == 0) {
        mbar_init(x_full, 1);
        mbar_init(&p_full[0], 1);
        mbar_init(&p_full[1], 1);
        mbar_init(mma_done, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    bool ok = true;

    if (tid == 0) {
        mbar_expect_tx(x_full, C::TILE);
        for (int p = 0; p < D / 64; ++p) tma_load_2d(X[0] + p * 16384, &mKt, 64 * p, h * Lp + J * BT, x_full);
        if (J + 1 < last) {  // P_{J+1} for the first transport step
            mbar_expect_tx(&p_full[0], C::PB);
            for (int p = 0; p < D / 64; ++p)
                tma_load_2d(Pb[0] + p * (D * 128), &mP, 64 * p, (h * nblk + J + 1) * D, &p_full[0]);
        }
        ok = mbar_wait(x_full, 0, WAIT_LIMIT_NS);
        if (ok) {
            for (int p = 0; p < D / 64; ++p) tma_store_2d(&mKh, 64 * p, pair_row(J + 1), X[0] + p * 16384);
            bulk_commit();
        }
    }
    const uint32_t idesc = idesc_f16(128, D, AB_F16, 0, 0);
    // step t transports the output of pair (I, J) into pair (I+1, J), I = J+1+t
    for (int I = J + 1; I < last; ++I) {
        const int t = I - J - 1;
        uint8_t *cur = X[t & 1], *nxt = X[(t + 1) & 1];
        if (tid == 0 && ok) {
            ok = mbar_wait(&p_full[t & 1], (t >> 1) & 1, WAIT_LIMIT_NS);
            if (ok && I + 1 < last) {  // prefetch P_{I+1}; its buffer's last reader has completed
                mbar_expect_tx(&p_full[(t + 1) & 1], C::PB);
                for (int p = 0; p < D / 64; ++p)
                    tma_load_2d(Pb[(t + 1) & 1] + p * (D * 128), &mP, 64 * p, (h * nblk + I + 1) * D,
                                &p_full[(t + 1) & 1]);
            }
            if (ok) {
                fence_after_sync();
                const uint32_t a0 = smem_u32(cur), b0 = smem_u32(Pb[t & 1]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t aoff = (kk / 4) * 16384 + (kk % 4) * 32;
                    const uint32_t boff = (kk / 4) * (D * 128) + (kk % 4) * 32;
                    mma_ss(tbase, desc_sw128(a0 + aoff, 16, 1024), desc_sw128(b0 + boff, 16, 1024),
                           idesc, kk > 0);
                }
                commit(mma_done);
            }
            // stores alternate between the two buffers: once at most one (the
            // latest, reading `cur`) is pending, `nxt` has been read out
            bulk_wait_read<1>();
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (!mbar_wait(mma_done, t & 1, WAIT_LIMIT_NS)) ok = false;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        fence_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            float v[32];
            tmem_ld32(tbase + c0 + lane_off, v);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint4 u;
                __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                for (int k = 0; k < 4; ++k) hh[k] = __floats2half2_rn(v[g * 8 + 2 * k], v[g * 8 + 2 * k + 1]);
                const int col = c0 + g * 8;
                *reinterpret_cast<uint4 *>(nxt + (col >> 6) * 16384 + sw128_offset(tid, col & 63)) = u;
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            for (int p = 0; p < D / 64; ++p) tma_store_2d(&mKh, 64 * p, pair_row(I + 1), nxt + p * 16384);
            bulk_commit();
        }
    }
    if (tid == 0) {
        bulk_wait_all();
        if (!ok && err) atomicCAS(err, 0, 4);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, C::TMEM_COLS);
}

template <int D>
cudaError_t launch_chain(const ChainArgs &c, int *err, cudaStream_t st)
{
    const int Lp = c.nblk * BT;
    const long long npairs = (long long)c.nblk * (c.nblk - 1) / 2;
    CUtensorMap mKt, mP, mKh;
    if (!make_map_2d(&mKt, c.Kt, F16, D, (uint64_t)c.nh * Lp, 128) ||
        !make_map_2d(&mP, c.Pm, F16, D, (uint64_t)c.nh * c.nblk * D, D) ||
        !make_map_2d(&mKh, c.Khat, F16, D, (uint64_t)c.nh * npairs * BT, 128))
        return cudaErrorInvalidValue;
    auto k = chain_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, ChainCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(c.nblk - 1, c.nh), 128, ChainCfg<D>::SMEM, st>>>(mKt, mP, mKh, c.nblk, npairs, err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

cudaError_t chain_tc(const ChainArgs &c, int d, int *err, cudaStream_t st)
{
    if (c.nblk < 2) return cudaSuccess;
    return d == 64 ? launch_chain<64>(c, err, st) : launch_chain<128>(c, err, st);
}

}  // namespace path
