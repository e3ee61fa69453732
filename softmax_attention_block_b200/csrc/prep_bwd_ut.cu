// Adjoint of the per-block UT prep on tcgen05 (tensor memory), head dim 64,
// bf16 inputs, from the per-half quantities the forward prep saved (UtSave).
//
// The attention backward hands over, per block, the adjoints of the
// boundary-adjusted queries / keys (dQtil, dKtil: 128 rows), of the block
// product (dP) and of the block's logits (dSd). One CTA per 64-position half
// block carries them to dq, dk, dw and dbeta:
//
// 1. The halves compose the block (Qtil[b] = Qtil_b P_a, Ktil[a] = Ktil_a P_b^T,
//    P = P_b P_a, Sd[b,a] = Qtil_b Ktil_a^T), so the block's adjoints become
//    per-half ones; each half's CTA forms its own:
//      half a: dQ_a = dQtil[a],  dK_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b,  dP_a = Qtil_b^T dQtil[b] + P_b^T dP
//      half b: dQ_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a,  dK_b = dKtil[b],  dP_b = dKtil[a]^T Ktil_a + dP P_a^T
// 2. With the half's UT transform (Paper-Notes "训练策略":
//    T^{-1} = (I + strictLower(D W W^T))^{-1} D, and X = (I + A)^{-1}) as the
//    forward saved it (What, U, -M, X), Qtil = Q - M What, Ktil = K - U^T W,
//    P = I - W^T What, Sd = lower(Q K^T - M U) and the half's adjoints dQ, dK,
//    dP, dS = dSd[h, h]:
//      dWhat = -M^T dQ - W dP,  dU = -W dK^T - M^T dS,  dM = lower(-dQ What^T - dS U^T)
//      dq = dQ + dS K + dM W
//      dR = X^T [dWhat | dU]                         (the transposed solve)
//      dA = strictLower(-(dR_w What^T + dR_n U^T)),  dN = strictLower(D dR_n), dG = strictLower(D dA)
//      dbeta_r = dR_w[r].W[r] + dR_n[r].N[r] + sum_c dA[r][c] G[r][c]    (G = W W^T, N = W K^T)
//      dk = dK + dS^T Q + dN^T W
//      dw = D dR_w - U dK - What dP^T + dM^T Q + dN K + (dG + dG^T) W
//
// The CTA is small enough for two per SM (106 KB of shared memory, 256
// tensor-memory columns). Products run on fp16 operands (the bf16 inputs are
// exact in fp16) with fp32 accumulation; dq, dk, dw add the fp32 adjoints dQ,
// dK (from global memory, or the composition's accumulator held in tensor
// memory) and D dR_w, and dbeta is formed from fp32 values. An M = 64
// accumulator sits in one of the two lane slots of a 64-column group (lane
// offsets 0 and 16, ut_tc.cuh), so a group holds two results.
#include "prep.cuh"
#include "runtime.cuh"
#include "ut_tc.cuh"

namespace path {

namespace {

using namespace tc;
using namespace uttc;

constexpr int NT = 256;
constexpr int SAVED_WORD = UT_SAVED_BYTE * 0x01010101;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// A 64 x 64 bf16 tile converted to fp16 in place (the products' operand type);
// the whole CTA, no barrier.
__device__ __forceinline__ void tile_bf16_to_f16(uint8_t *tile)
{
    const int t = threadIdx.x, row = t >> 2, c = (t & 3) * 16;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + sw128_offset(row, c + 8 * j));
        uint4 u = *p;
        __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&u);
        __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) hh[i] = __float22half2_rn(__bfloat1622float2(b[i]));
        *p = u;
    }
}

#define ISSUE(...)                 \
    do {                           \
        if (ok && warp == 0) {     \
            fence_after_sync();    \
            if (lane == 0) {       \
                __VA_ARGS__;       \
                commit(bar);       \
            }                      \
            __syncwarp();          \
        }                          \
    } while (0)

// shared-memory tiles (8 KB each)
enum {
    U_W = 0, U_K = 1,  // [W; K] is one 128-row operand
    U_Q = 2,
    U_M = 3,           // M (saved as -M) -> dM
    U_WH = 4,          // What
    U_U = 5,
    U_X = 6,           // X -> dN
    // the composition's operands, then the half's adjoints over them
    U_C0 = 7,          // dKtil[a] (half a) / dQtil[b] (half b) -> dQ -> dWhat -> dR_w
    U_C1 = 8,          // P_b / P_a -> dK
    U_C2 = 9,          // dSd[b, a] -> dP of the half
    U_C3 = 10,         // Qtil_b / Ktil_a -> dS -> dG
    U_C4 = 11,         // dQtil[b] / dKtil[a] -> dU -> dR_n
    U_C5 = 12,         // dP (the block's)
    U_NTILES = 13,
    U_DQ = U_C0, U_DK = U_C1, U_DP = U_C2, U_DS = U_C3, U_DU = U_C4,
};
constexpr int U_BETA_OFF = U_NTILES * TILE;      // [64] beta
constexpr int U_PART_OFF = U_BETA_OFF + 64 * 4;  // [4][64] dbeta partial sums
constexpr int U_BAR_OFF = U_PART_OFF + 4 * 64 * 4;
constexpr int U_SMEM = U_BAR_OFF + 64 + 1024;
static_assert(2 * (U_SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
// tensor-memory 64-column groups; (slot, group) of each result
constexpr int G0 = 0, G1 = 64, G2 = 128, G3 = 192;
// CA: the composition's results in G3: half a dK_a (1) and dP_a (0), half b dQ_b (0)
//     and dP_b (1); dK_a / dQ_b held there until dk / dq add it
// B1: dWhat' (0, G0), dU' (1, G0), dM' (0, G1); B2: dR_w (0, G2), dR_n (1, G2) held to
// the end, dS K + dM W (0, G0); B3: dA' (0, G0), dS^T Q + dN^T W (1, G0), G (0, G1),
// N (1, G1); B4: dw's positive terms (0, G0), its negative terms (0, G1)

template <typename TO>
__global__ void __launch_bounds__(NT, 2)
    ut_adj64_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mQ,
                    const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mH,
                    const __grid_constant__ CUtensorMap mB, const float *beta, int L, int nblk,
                    const float *dQt, const float *dKt, const float *dPm, const float *dSd, TO *dq,
                    TO *dk, TO *dw, float *dbeta, const int *saved, int *err)
{
    if (*saved != SAVED_WORD) {  // nothing to read: record it, write nothing
        if (threadIdx.x == 0 && err) atomicCAS(err, 0, ERR_UT_NOT_SAVED);
        return;
    }
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    auto tile = [&](int i) { return sm + i * TILE; };
    const uint32_t s0 = smem_u32(sm);
    auto ta = [&](int i) { return s0 + (uint32_t)i * TILE; };
    float *sB = reinterpret_cast<float *>(sm + U_BETA_OFF);
    float *sPart = reinterpret_cast<float *>(sm + U_PART_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + U_BAR_OFF);  // [0] loads, [1] MMA
    uint64_t *bar = &bars[1];
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int J = blockIdx.x >> 1, hf = blockIdx.x & 1, hd = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long blk = (long long)hd * nblk + J;
    const int prow0 = J * BT + hf * HB;                          // half's first position
    const long long brow = (long long)hd * nblk * BT + (long long)J * BT;  // block's first row in [nh, Lp]
    const int srow = (int)((blk * 2 + hf) * HB);                 // in the per-half save arrays
    // the save's What, U, X, -M ([nb 2 64, 64] each, stacked at hstride rows) and
    // Kta, Qtb, Pa, Pb ([nb 64, 64] each, bstride rows)
    const int hstride = nblk * gridDim.y * 2 * HB, bstride = nblk * gridDim.y * HB;
    const float *dsdb = dSd + blk * BT * BT;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        mbar_expect_tx(&bars[0], 9 * TILE);
        tma_load_3d(tile(U_W), &mW, 0, prow0, hd, &bars[0]);
        tma_load_3d(tile(U_K), &mK, 0, prow0, hd, &bars[0]);
        tma_load_3d(tile(U_Q), &mQ, 0, prow0, hd, &bars[0]);
        tma_load_2d(tile(U_WH), &mH, 0, srow, &bars[0]);
        tma_load_2d(tile(U_U), &mH, 0, hstride + srow, &bars[0]);
        tma_load_2d(tile(U_X), &mH, 0, 2 * hstride + srow, &bars[0]);
        tma_load_2d(tile(U_M), &mH, 0, 3 * hstride + srow, &bars[0]);
        // half a: P_b (index 3) and Qtil_b (1); half b: P_a (2) and Ktil_a (0)
        tma_load_2d(tile(U_C1), &mB, 0, (hf ? 2 : 3) * bstride + (int)blk * HB, &bars[0]);
        tma_load_2d(tile(U_C3), &mB, 0, (hf ? 0 : 1) * bstride + (int)blk * HB, &bars[0]);
    }
    if (warp == 0) tmem_alloc(tslot, 256);
    const Me me;
    const int s = me.h, r = me.r, c0 = 32 * me.cg;
    // the fp32 row the half itself adds rather than forms: dQ_a (half a, for dq, slot 0)
    // or dK_b (half b, for dk, slot 1); in flight from here to its use
    float xl[32];
    if (s == hf)
        ld_global((hf ? dKt + (brow + HB + r) * HB : dQt + (brow + r) * HB) + c0, xl);
    {   // the composition's fp32 operands as fp16 tiles
        uint8_t *const t[4] = {tile(U_C0), tile(U_C2), tile(U_C4), tile(U_C5)};
        const float *const src[4] = {hf ? dQt + (brow + HB) * HB : dKt + brow * HB,
                                     dsdb + (long long)HB * BT,
                                     hf ? dKt + brow * HB : dQt + (brow + HB) * HB,
                                     dPm + blk * HB * HB};
        const int ld[4] = {HB, BT, HB, HB};
        tiles_from_f32(t, src, ld);
    }
    if (tid < HB) {
        const int p = prow0 + tid;
        sB[tid] = p < L ? beta[(long long)hd * L + p] : 0.f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = mbar_wait(&bars[0], 0, WAIT_LIMIT_NS);
    if (ok) {  // W, K, Q (bf16 inputs, exact in fp16) beside the fp16 operands; M from the saved -M
        tile_bf16_to_f16(tile(U_W));
        tile_bf16_to_f16(tile(U_K));
        tile_bf16_to_f16(tile(U_Q));
        negate_tile(tile(U_M));
    }
    fence_async_smem();
    fence_before_sync();
    ok = __syncthreads_and(ok);

    const float br = sB[r];
    const int pos = prow0 + r;
    const bool valid = pos < L;
    const long long grow = (long long)hd * L + pos;  // row in [nh, L]
    uint32_t phase = 0;
    auto sync_operands = [&]() {
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok);
    };
    auto wait_mma = [&]() {
        if (ok && !mbar_wait(bar, phase, WAIT_LIMIT_NS)) ok = false;
        phase ^= 1;
        fence_after_sync();
    };
    float v[32], x[32];

    // ---- CA: this half's adjoints from the block's
    ISSUE({
        if (hf == 0) {
            // dK_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b; dP_a = Qtil_b^T dQtil[b] + P_b^T dP
            mma64(dst(tbase, 1, G3), ta(U_C0), A_N, ta(U_C1), B_N, 1, TILE, false);
            mma64(dst(tbase, 1, G3), ta(U_C2), A_T, ta(U_C3), B_N, 1, TILE, true);
            mma64(dst(tbase, 0, G3), ta(U_C3), A_T, ta(U_C4), B_N, 1, TILE, false);
            mma64(dst(tbase, 0, G3), ta(U_C1), A_T, ta(U_C5), B_N, 1, TILE, true);
        } else {
            // dQ_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a; dP_b = dKtil[a]^T Ktil_a + dP P_a^T
            mma64(dst(tbase, 0, G3), ta(U_C0), A_N, ta(U_C1), B_T, 1, TILE, false);
            mma64(dst(tbase, 0, G3), ta(U_C2), A_N, ta(U_C3), B_N, 1, TILE, true);
            mma64(dst(tbase, 1, G3), ta(U_C4), A_T, ta(U_C3), B_N, 1, TILE, false);
            mma64(dst(tbase, 1, G3), ta(U_C5), A_N, ta(U_C1), B_T, 1, TILE, true);
        }
    });
    // meanwhile: dS = dSd[h, h] (fp32) into registers, one thread per 16 values
    float4 dsr[4];
    {
        const float *src = dsdb + (long long)hf * HB * BT + hf * HB + (long long)(tid >> 2) * BT + (tid & 3) * 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) dsr[i] = reinterpret_cast<const float4 *>(src)[i];
    }
    wait_mma();
    if (ok) {
        // the composition's operands are read: their tiles take the half's adjoints
        me.ld(tbase, G3, v);
        if (s == hf)  // dQ_a from global (half a), dK_b likewise (half b)
            st_tile_f16(tile(hf ? U_DK : U_DQ), r, c0, xl);
        else          // dK_a (half a), dQ_b (half b): this half's composition result
            st_tile_f16(tile(hf ? U_DQ : U_DK), r, c0, v);
        // dP_h: slot 0 in half a, slot 1 in half b
        if (s == hf) st_tile_f16(tile(U_DP), r, c0, v);
        const int row = tid >> 2, c = (tid & 3) * 16;
        const float *f = reinterpret_cast<const float *>(dsr);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint4 u;
            __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) hh[i] = __floats2half2_rn(f[8 * j + 2 * i], f[8 * j + 2 * i + 1]);
            *reinterpret_cast<uint4 *>(tile(U_DS) + sw128_offset(row, c + 8 * j)) = u;
        }
    }
    sync_operands();

    // ---- B1: dWhat' = M^T dQ + W dP, dU' = W dK^T + M^T dS, dM' = dQ What^T + dS U^T
    ISSUE({
        mma64(dst(tbase, 0, G0), ta(U_M), A_T, ta(U_DQ), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, G0), ta(U_W), A_N, ta(U_DP), B_N, 1, TILE, true);
        mma64(dst(tbase, 1, G0), ta(U_W), A_N, ta(U_DK), B_T, 1, TILE, false);
        mma64(dst(tbase, 1, G0), ta(U_M), A_T, ta(U_DS), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, G1), ta(U_DQ), A_N, ta(U_WH), B_T, 1, TILE, false);
        mma64(dst(tbase, 0, G1), ta(U_DS), A_N, ta(U_U), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, G0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(s ? U_DU : U_DQ), r, c0, v);  // dU (slot 1) or dWhat (slot 0, over dQ)
        me.ld(tbase, G1, v);
        if (s == 0) {  // dM = lower(-dM'), over M
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = c0 + j <= r ? -v[j] : 0.f;
            st_tile_f16(tile(U_M), r, c0, v);
        }
    }
    sync_operands();

    // ---- B2: dR = X^T [dWhat | dU], dS K + dM W
    ISSUE({
        mma64(dst(tbase, 0, G2), ta(U_X), A_T, ta(U_DQ), B_N, 1, TILE, false);
        mma64(dst(tbase, 1, G2), ta(U_X), A_T, ta(U_DU), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, G0), ta(U_DS), A_N, ta(U_K), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, G0), ta(U_M), A_N, ta(U_W), B_N, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, G2, v);
        st_tile_f16(tile(s ? U_DU : U_DQ), r, c0, v);  // dR_n over dU (slot 1), dR_w over dWhat
        if (s == 1) {  // dN = strictLower(D dR_n), over X
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = c0 + j < r ? br * v[j] : 0.f;
            st_tile_f16(tile(U_X), r, c0, v);
        }
        me.ld(tbase, G0, v);  // dq = dQ + dS K + dM W (slot 0)
        me.ld(tbase, G3, x);  // dQ_b in half b (slot 0)
        if (s == 0 && valid) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += hf ? x[j] : xl[j];
            st_global(dq + grow * HB + c0, v);
        }
    }
    sync_operands();

    // ---- B3: dA' = dR_w What^T + dR_n U^T, dS^T Q + dN^T W, and G = W W^T, N = W K^T again
    ISSUE({
        mma64(dst(tbase, 0, G0), ta(U_DQ), A_N, ta(U_WH), B_T, 1, TILE, false);
        mma64(dst(tbase, 0, G0), ta(U_DU), A_N, ta(U_U), B_T, 1, TILE, true);
        mma64(dst(tbase, 1, G0), ta(U_DS), A_T, ta(U_Q), B_N, 1, TILE, false);
        mma64(dst(tbase, 1, G0), ta(U_X), A_T, ta(U_W), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, G1), ta(U_W), A_N, ta(U_W), B_T, 1, TILE, false);
        mma64(dst(tbase, 1, G1), ta(U_W), A_N, ta(U_K), B_T, 1, TILE, false);
    });
    wait_mma();
    if (ok) {
        // dbeta_r partials: slot 0 dR_w[r].W[r] + sum_c dA[r][c] G[r][c] (and dG =
        // strictLower(D dA) over dS); slot 1 dR_n[r].N[r] (N = strictLower(W K^T))
        float sum = 0.f;
        me.ld(tbase, G2, v);
        me.ld(tbase, G1, x);
        if (s == 0) {
            float wv[32];
            ld_tile_f16(tile(U_W), r, c0, wv);
#pragma unroll
            for (int j = 0; j < 32; ++j) sum = fmaf(v[j], wv[j], sum);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) sum = fmaf(v[j], c0 + j < r ? x[j] : 0.f, sum);
        }
        me.ld(tbase, G0, v);
        if (s == 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float da = c0 + j < r ? -v[j] : 0.f;  // dA = strictLower(-dA')
                sum = fmaf(da, x[j], sum);
                v[j] = br * da;
            }
            st_tile_f16(tile(U_DS), r, c0, v);
        }
        sPart[(2 * s + me.cg) * HB + r] = sum;
        me.ld(tbase, G3, x);  // dK_a in half a (slot 1)
        if (s == 1 && valid) {  // dk = dK + dS^T Q + dN^T W
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += hf ? xl[j] : x[j];
            st_global(dk + grow * HB + c0, v);
        }
    }
    sync_operands();
    if (ok && tid < HB && prow0 + tid < L)
        dbeta[(long long)hd * L + prow0 + tid] =
            sPart[tid] + sPart[HB + tid] + sPart[2 * HB + tid] + sPart[3 * HB + tid];

    // ---- B4: dw = D dR_w + (dM^T Q + dN K + dG W + dG^T W) - (U dK + What dP^T)
    ISSUE({
        mma64(dst(tbase, 0, G0), ta(U_M), A_T, ta(U_Q), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, G0), ta(U_X), A_N, ta(U_K), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, G0), ta(U_DS), A_N, ta(U_W), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, G0), ta(U_DS), A_T, ta(U_W), B_N, 1, TILE, true);
        mma64(dst(tbase, 0, G1), ta(U_U), A_N, ta(U_DK), B_N, 1, TILE, false);
        mma64(dst(tbase, 0, G1), ta(U_WH), A_N, ta(U_DP), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, G0, v);
        me.ld(tbase, G1, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] -= x[j];
        me.ld(tbase, G2, x);
        if (s == 0 && valid) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaf(br, x[j], v[j]);
            st_global(dw + grow * HB + c0, v);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 26);
    if (warp == 0) tmem_dealloc(tbase, 256);
}

#undef ISSUE

template <typename TO>
cudaError_t launch_adj(const CUtensorMap *m, const PrepDims &Dm, const PrepInputs &in,
                       const PrepGrads &g, const int *saved, int *err, cudaStream_t st)
{
    auto k = ut_adj64_kernel<TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, U_SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(2 * Dm.nblk, Dm.nh), NT, U_SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], in.beta, Dm.L, Dm.nblk,
                                                     g.dQt, g.dKt, g.dPm, g.dSd, static_cast<TO *>(g.dq),
                                                     static_cast<TO *>(g.dk), static_cast<TO *>(g.dw),
                                                     g.dbeta, saved, err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool prep_backward_ut_supported(const PrepDims &Dm, const PrepInputs &in)
{
    // the save area's stacked maps index up to 4 nh nblk 128 rows (int32)
    return prep_forward_ut_supported(Dm, in) && (long long)Dm.nh * Dm.nblk * 4 * BT < (1LL << 31);
}

cudaError_t prep_backward_ut(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g,
                             const UtSave &sv, const int *saved, int *err, cudaStream_t st)
{
    if (!prep_backward_ut_supported(Dm, in)) return cudaErrorInvalidValue;
    // What, U, X, M and Kta, Qtb, Pa, Pb lie back to back (carve_ut_save): one map each
    const uint64_t nb = (uint64_t)Dm.nh * Dm.nblk, hsz = nb * 2 * HB * HB, bsz = nb * HB * HB;
    if (sv.U != sv.What + hsz || sv.X != sv.U + hsz || sv.M != sv.X + hsz || sv.Qtb != sv.Kta + bsz ||
        sv.Pa != sv.Qtb + bsz || sv.Pb != sv.Pa + bsz)
        return cudaErrorInvalidValue;
    CUtensorMap m[5];
    if (!make_map_3d(&m[0], in.w, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[1], in.q, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[2], in.k, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_2d(&m[3], sv.What, F16, HB, 4 * nb * 2 * HB, HB) ||
        !make_map_2d(&m[4], sv.Kta, F16, HB, 4 * nb * HB, HB))
        return cudaErrorInvalidValue;
    if (Dm.odt == F32) return launch_adj<float>(m, Dm, in, g, saved, err, st);
    return launch_adj<bf16>(m, Dm, in, g, saved, err, st);
}

}  // namespace path
