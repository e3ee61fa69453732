// Adjoint of the head-dim-128 UT prep (prep_fwd_ut128.cu) on tcgen05, bf16
// inputs, from the per-half quantities that forward saved (UtSave).
//
// The attention backward hands over, per block, the adjoints of the
// boundary-adjusted queries / keys (dQtil, dKtil: 128 rows), of the block
// product (dP) and of the block's logits (dSd). Two kernels carry them to dq,
// dk, dw and dbeta:
//
// 1. compose_adj128_kernel, one CTA per block: the halves compose the block
//    (Qtil[b] = Qtil_b P_a, Ktil[a] = Ktil_a P_b^T, P = P_b P_a,
//    Sd[b,a] = Qtil_b Ktil_a^T), so the block's adjoints become per-half ones:
//      dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a,  dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b,
//      dP_a = Qtil_b^T dQtil[b] + P_b^T dP,          dP_b = dKtil[a]^T Ktil_a + dP P_a^T
//    (dQtil_a = dQtil[a], dKtil_b = dKtil[b]). dQtil_b and dKtil_a overwrite
//    dQtil[b] and dKtil[a] (fp32); dP_a, dP_b go to the save area (fp16).
// 2. ut_adj128_kernel, one CTA per half block: with Qtil = Q - M What,
//    Ktil = K - U^T W, P = I - W^T What, Sd = lower(Q K^T - M U) and the
//    half's adjoints dQ, dK, dP, dS (Paper-Notes "训练策略" for the transform
//    T^{-1} = (I + strictLower(D W W^T))^{-1} D, X = (I + A)^{-1}):
//      dWhat = -M^T dQ - W dP,  dU = -W dK^T - M^T dS,  dM = lower(-dQ What^T - dS U^T)
//      dq = dQ + dS K + dM W
//      dR = X^T [dWhat | dU]
//      dA = strictLower(-(dR_w What^T + dR_n U^T)),  dN = strictLower(D dR_n), dG = strictLower(D dA)
//      dbeta_r = dR_w[r].W[r] + dR_n[r].N[r] + sum_c dA[r][c] G[r][c]    (G = W W^T, N = W K^T)
//      dk = dK + dS^T Q + dN^T W
//      dw = D dR_w - U dK - What dP^T + dM^T Q + dN K + (dG + dG^T) W
//
// Products are M = 64 MMAs on fp16 operands with fp32 accumulation. In the
// per-half kernel the two lane slots of tensor memory (lane offsets 0 and 16,
// ut_tc.cuh) hold the two 64-column halves of a 128-wide result, or two
// different 64 x 64 results, so every thread of the epilogue has a row.
#include "prep.cuh"
#include "runtime.cuh"
#include "ut_tc.cuh"

namespace path {

namespace {

using namespace tc;
using namespace uttc;

constexpr int NT = 256;
constexpr int DH = 128;  // head dim
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

// ---------------------------------------------------------------------------
// 1. composition adjoint
// shared-memory tiles (8 KB each)
enum {
    CA_KTA = 0,    // Ktil_a, 2 column tiles
    CA_QTB = 2,    // Qtil_b
    CA_PA = 4,     // P_a: tile 4 + 2 cb + rb (its two row blocks adjacent: a 128-row K-major B)
    CA_PB = 8,     // P_b: tile 8 + 2 rb + cb (row blocks as K-chunks of an MN-major B)
    CA_DKA = 12,   // dKtil[a]
    CA_DQB = 14,   // dQtil[b]
    CA_DSBA = 16,  // dSd[b, a]
    CA_DP = 17,    // dP: tile 17 + 2 rb + cb
    CA_NTILES = 21,
};
constexpr int CA_BAR_OFF = CA_NTILES * TILE;
constexpr int CA_SMEM = CA_BAR_OFF + 64 + 1024;
// tensor memory: half a's lanes dKtil_a | dP_a, half b's dQtil_b | dP_b
constexpr int CA_C = 0, CA_CP = 128;  // 128-wide results; dP row block rb at CA_CP + 128 rb

__global__ void __launch_bounds__(NT, 1)
    compose_adj128_kernel(const __grid_constant__ CUtensorMap mKta, const __grid_constant__ CUtensorMap mQtb,
                          const __grid_constant__ CUtensorMap mPa, const __grid_constant__ CUtensorMap mPb,
                          int nblk, float *dQt, float *dKt, const float *dPm, const float *dSd, f16 *dPs,
                          const int *saved, int *err)
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
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CA_BAR_OFF);  // [0] loads, [1] MMA
    uint64_t *bar = &bars[1];
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int J = blockIdx.x, hd = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long blk = (long long)hd * nblk + J;
    const long long brow = (long long)hd * nblk * BT + (long long)J * BT;  // block's first row in [nh, Lp]

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        mbar_expect_tx(&bars[0], 12 * TILE);
        for (int c = 0; c < 2; ++c) {
            tma_load_2d(tile(CA_KTA + c), &mKta, 64 * c, (int)(blk * HB), &bars[0]);
            tma_load_2d(tile(CA_QTB + c), &mQtb, 64 * c, (int)(blk * HB), &bars[0]);
            for (int rb = 0; rb < 2; ++rb) {
                tma_load_2d(tile(CA_PA + 2 * c + rb), &mPa, 64 * c, (int)(blk * DH + 64 * rb), &bars[0]);
                tma_load_2d(tile(CA_PB + 2 * rb + c), &mPb, 64 * c, (int)(blk * DH + 64 * rb), &bars[0]);
            }
        }
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    // the fp32 adjoints as fp16 operands
    const float *dsdb = dSd + blk * BT * BT;
    const float *dpb = dPm + blk * DH * DH;
    {   // dKtil[a], dQtil[b], dSd[b, a]
        uint8_t *const t[5] = {tile(CA_DKA), tile(CA_DKA + 1), tile(CA_DQB), tile(CA_DQB + 1), tile(CA_DSBA)};
        const float *const src[5] = {dKt + brow * DH, dKt + brow * DH + 64, dQt + (brow + HB) * DH,
                                     dQt + (brow + HB) * DH + 64, dsdb + (long long)HB * BT};
        const int ld[5] = {DH, DH, DH, DH, BT};
        tiles_from_f32(t, src, ld);
    }
    {   // dP
        uint8_t *const t[4] = {tile(CA_DP), tile(CA_DP + 1), tile(CA_DP + 2), tile(CA_DP + 3)};
        const float *const src[4] = {dpb, dpb + 64, dpb + 64 * DH, dpb + 64 * DH + 64};
        const int ld[4] = {DH, DH, DH, DH};
        tiles_from_f32(t, src, ld);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = mbar_wait(&bars[0], 0, WAIT_LIMIT_NS);
    ok = __syncthreads_and(ok);

    ISSUE({
        for (int k = 0; k < 2; ++k) {
            // half a: dKtil_a = dKtil[a] P_b + dSd[b,a]^T Qtil_b
            mma64(dst(tbase, 0, CA_C), ta(CA_DKA + k), A_N, ta(CA_PB + 2 * k), B_N, 2, TILE, k > 0);
            // half b: dQtil_b = dQtil[b] P_a^T + dSd[b,a] Ktil_a
            mma64(dst(tbase, 1, CA_C), ta(CA_DQB + k), A_N, ta(CA_PA + 2 * k), B_T, 2, TILE, k > 0);
        }
        mma64(dst(tbase, 0, CA_C), ta(CA_DSBA), A_T, ta(CA_QTB), B_N, 2, TILE, true);
        mma64(dst(tbase, 1, CA_C), ta(CA_DSBA), A_N, ta(CA_KTA), B_N, 2, TILE, true);
        for (int rb = 0; rb < 2; ++rb) {
            const int col = CA_CP + 128 * rb;
            // dP_a = Qtil_b^T dQtil[b] + P_b^T dP   (rows 64 rb..)
            mma64(dst(tbase, 0, col), ta(CA_QTB + rb), A_T, ta(CA_DQB), B_N, 2, TILE, false);
            // dP_b = dKtil[a]^T Ktil_a + dP P_a^T
            mma64(dst(tbase, 1, col), ta(CA_DKA + rb), A_T, ta(CA_KTA), B_N, 2, TILE, false);
            for (int k = 0; k < 2; ++k) {
                mma64(dst(tbase, 0, col), ta(CA_PB + 2 * k + rb), A_T, ta(CA_DP + 2 * k), B_N, 2, TILE, true);
                mma64(dst(tbase, 1, col), ta(CA_DP + 2 * rb + k), A_N, ta(CA_PA + 2 * k), B_T, 2, TILE, true);
            }
        }
    });
    uint32_t phase = 0;
    if (ok && !mbar_wait(bar, phase, WAIT_LIMIT_NS)) ok = false;
    fence_after_sync();
    if (ok) {
        const Me me;
        const int h = me.h, r = me.r, c0 = 32 * me.cg;
        float v[32];
        // half a: dKtil_a over dKtil[a]; half b: dQtil_b over dQtil[b]
        float *drow = h ? dQt + (brow + HB + r) * DH : dKt + (brow + r) * DH;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            me.ld(tbase, CA_C + 64 * c, v);
            st_global(drow + 64 * c + c0, v);
        }
        f16 *prow = dPs + ((blk * 2 + h) * DH + r) * DH;
#pragma unroll 1
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                me.ld(tbase, CA_CP + 128 * rb + 64 * c, v);
                st_global(prow + 64 * rb * DH + 64 * c + c0, v);
            }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 24);
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ---------------------------------------------------------------------------
// 2. per-half UT adjoint
enum {
    U_W = 0,    // W.c at 2c, K.c at 2c + 1 ([W.c; K.c] is one 128-row B)
    U_Q = 4,    // Q, 2 tiles
    U_M = 6,    // M -> dM
    U_WH = 7,   // What, 2 tiles
    U_U = 9,    // U
    U_X = 10,   // X -> dN
    U_DQ = 11,  // dQ (2) -> dWhat -> dR_w
    U_DK = 13,  // dK (2)
    U_DS = 15,  // dS -> dG
    U_DP = 16,  // dP: tile 16 + 2 rb + cb
    U_DU = 20,  // dU -> dR_n
    U_NTILES = 21,
};
constexpr int U_BETA_OFF = U_NTILES * TILE;      // [64] beta
constexpr int U_PART_OFF = U_BETA_OFF + 64 * 4;  // [4][64] dbeta partial sums
constexpr int U_BAR_OFF = U_PART_OFF + 4 * 64 * 4;
constexpr int U_SMEM = U_BAR_OFF + 64 + 1024;
// tensor-memory columns; "both": slot s holds column half s of a 128-wide result
constexpr int UC_B1W = 0;    // dWhat' (both)
constexpr int UC_B1S = 64;   // slot 0: dU', slot 1: dM'
constexpr int UC_DRW = 0;    // dR_w (both), held to the end
constexpr int UC_DRN = 64;   // slot 0: dR_n, held to the end
constexpr int UC_DQ = 128;   // dS K + dM W (both)
constexpr int UC_DA = 192;   // slot 0: dA'
constexpr int UC_DK = 256;   // dS^T Q + dN^T W (both)
constexpr int UC_GN = 320;   // slot 0: G | N
constexpr int UC_W1 = 128;   // dw: positive terms (both)
constexpr int UC_W2 = 192;   // dw: negative terms (both)

template <typename TO>
__global__ void __launch_bounds__(NT, 1)
    ut_adj128_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mQ,
                     const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mWh,
                     const __grid_constant__ CUtensorMap mU, const __grid_constant__ CUtensorMap mX,
                     const __grid_constant__ CUtensorMap mM, const __grid_constant__ CUtensorMap mDP,
                     const float *beta, int L, int nblk, const float *dQt, const float *dKt,
                     const float *dSd, TO *dq, TO *dk, TO *dw, float *dbeta, const int *saved, int *err)
{
    if (*saved != SAVED_WORD) {
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
    const int prow0 = J * BT + hf * HB;                                  // half's first position
    const long long hrow = (long long)hd * nblk * BT + prow0;            // and its row in [nh, Lp]
    const int srow = (int)((blk * 2 + hf) * HB);                         // in the per-half save arrays

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        mbar_expect_tx(&bars[0], 15 * TILE);
        for (int c = 0; c < 2; ++c) {
            tma_load_3d(tile(U_W + 2 * c), &mW, 64 * c, prow0, hd, &bars[0]);
            tma_load_3d(tile(U_W + 2 * c + 1), &mK, 64 * c, prow0, hd, &bars[0]);
            tma_load_3d(tile(U_Q + c), &mQ, 64 * c, prow0, hd, &bars[0]);
            tma_load_2d(tile(U_WH + c), &mWh, 64 * c, srow, &bars[0]);
            for (int rb = 0; rb < 2; ++rb)
                tma_load_2d(tile(U_DP + 2 * rb + c), &mDP, 64 * c, 2 * srow + 64 * rb, &bars[0]);
        }
        tma_load_2d(tile(U_U), &mU, 0, srow, &bars[0]);
        tma_load_2d(tile(U_X), &mX, 0, srow, &bars[0]);
        tma_load_2d(tile(U_M), &mM, 0, srow, &bars[0]);
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    {   // dQ, dK and dS = dSd[h, h] as fp16 operands
        uint8_t *const t[5] = {tile(U_DQ), tile(U_DQ + 1), tile(U_DK), tile(U_DK + 1), tile(U_DS)};
        const float *const src[5] = {dQt + hrow * DH, dQt + hrow * DH + 64, dKt + hrow * DH, dKt + hrow * DH + 64,
                                     dSd + blk * BT * BT + (long long)hf * HB * BT + hf * HB};
        const int ld[5] = {DH, DH, DH, DH, BT};
        tiles_from_f32(t, src, ld);
    }
    if (tid < HB) {
        const int p = prow0 + tid;
        sB[tid] = p < L ? beta[(long long)hd * L + p] : 0.f;
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = mbar_wait(&bars[0], 0, WAIT_LIMIT_NS);
    if (ok) {  // W, K, Q (bf16 inputs, exact in fp16) beside the fp16 operands; M from the saved -M
        for (int i = 0; i < 4; ++i) tile_bf16_to_f16(tile(U_W + i));
        for (int c = 0; c < 2; ++c) tile_bf16_to_f16(tile(U_Q + c));
        negate_tile(tile(U_M));
    }
    fence_async_smem();
    ok = __syncthreads_and(ok);

    // epilogue place: slot s (lane offset 16 s), row r, 32 columns c0.. of each 64
    const Me me;
    const int s = me.h, r = me.r, c0 = 32 * me.cg;
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

    // ---- B1: dWhat' = M^T dQ + W dP, dU' = W dK^T + M^T dS, dM' = dQ What^T + dS U^T
    ISSUE({
        for (int c = 0; c < 2; ++c) {
            mma64(dst(tbase, c, UC_B1W), ta(U_M), A_T, ta(U_DQ + c), B_N, 1, TILE, false);
            for (int k = 0; k < 2; ++k)
                mma64(dst(tbase, c, UC_B1W), ta(U_W + 2 * k), A_N, ta(U_DP + 2 * k + c), B_N, 1, TILE, true);
        }
        for (int k = 0; k < 2; ++k) {
            mma64(dst(tbase, 0, UC_B1S), ta(U_W + 2 * k), A_N, ta(U_DK + k), B_T, 1, TILE, k > 0);
            mma64(dst(tbase, 1, UC_B1S), ta(U_DQ + k), A_N, ta(U_WH + k), B_T, 1, TILE, k > 0);
        }
        mma64(dst(tbase, 0, UC_B1S), ta(U_M), A_T, ta(U_DS), B_N, 1, TILE, true);
        mma64(dst(tbase, 1, UC_B1S), ta(U_DS), A_N, ta(U_U), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, UC_B1W, v);  // dWhat = -dWhat', column half s, over dQ's tile s
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(U_DQ + s), r, c0, v);
        me.ld(tbase, UC_B1S, v);
        if (s == 0) {  // dU = -dU'
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = -v[j];
            st_tile_f16(tile(U_DU), r, c0, v);
        } else {       // dM = lower(-dM'), over M
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = c0 + j <= r ? -v[j] : 0.f;
            st_tile_f16(tile(U_M), r, c0, v);
        }
    }
    sync_operands();

    // ---- B2: dR = X^T [dWhat | dU], dS K + dM W
    ISSUE({
        for (int c = 0; c < 2; ++c) {
            mma64(dst(tbase, c, UC_DRW), ta(U_X), A_T, ta(U_DQ + c), B_N, 1, TILE, false);
            mma64(dst(tbase, c, UC_DQ), ta(U_DS), A_N, ta(U_W + 2 * c + 1), B_N, 1, TILE, false);
            mma64(dst(tbase, c, UC_DQ), ta(U_M), A_N, ta(U_W + 2 * c), B_N, 1, TILE, true);
        }
        mma64(dst(tbase, 0, UC_DRN), ta(U_X), A_T, ta(U_DU), B_N, 1, TILE, false);
    });
    ld_global(dQt + (hrow + r) * DH + 64 * s + c0, x);  // in flight during the MMAs
    wait_mma();
    if (ok) {
        me.ld(tbase, UC_DQ, v);  // dq = dQ + dS K + dM W (column half s)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += x[j];
        if (valid) st_global(dq + grow * DH + 64 * s + c0, v);
        me.ld(tbase, UC_DRW, v);
        st_tile_f16(tile(U_DQ + s), r, c0, v);  // dR_w over dWhat
        me.ld(tbase, UC_DRN, v);
        if (s == 0) {
            st_tile_f16(tile(U_DU), r, c0, v);  // dR_n over dU
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = c0 + j < r ? br * v[j] : 0.f;
            st_tile_f16(tile(U_X), r, c0, v);   // dN = strictLower(D dR_n), over X
        }
    }
    sync_operands();

    // ---- B3: dA' = dR_w What^T + dR_n U^T, dS^T Q + dN^T W, and G | N = W [W; K]^T again
    ISSUE({
        for (int k = 0; k < 2; ++k) {
            mma64(dst(tbase, 0, UC_DA), ta(U_DQ + k), A_N, ta(U_WH + k), B_T, 1, TILE, k > 0);
            mma64(dst(tbase, 0, UC_GN), ta(U_W + 2 * k), A_N, ta(U_W + 2 * k), B_T, 2, TILE, k > 0);
        }
        mma64(dst(tbase, 0, UC_DA), ta(U_DU), A_N, ta(U_U), B_T, 1, TILE, true);
        for (int c = 0; c < 2; ++c) {
            mma64(dst(tbase, c, UC_DK), ta(U_DS), A_T, ta(U_Q + c), B_N, 1, TILE, false);
            mma64(dst(tbase, c, UC_DK), ta(U_X), A_T, ta(U_W + 2 * c), B_N, 1, TILE, true);
        }
    });
    float xk[32];
    ld_global(dKt + (hrow + r) * DH + 64 * s + c0, xk);  // in flight during the MMAs
    wait_mma();
    if (ok) {
        // dbeta_r partials: dR_w[r].W[r] over column half s; slot 0 also
        // dR_n[r].N[r] + sum_c dA[r][c] G[r][c] and dG = strictLower(D dA)
        float sum = 0.f;
        me.ld(tbase, UC_DRW, v);
        ld_tile_f16(tile(U_W + 2 * s), r, c0, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) sum = fmaf(v[j], x[j], sum);
        me.ld(tbase, UC_DRN, v);
        me.ld(tbase, UC_GN + 64, x);
        if (s == 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) sum = fmaf(v[j], c0 + j < r ? x[j] : 0.f, sum);
        }
        me.ld(tbase, UC_DA, v);
        me.ld(tbase, UC_GN, x);
        if (s == 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float da = c0 + j < r ? -v[j] : 0.f;  // dA = strictLower(-dA')
                sum = fmaf(da, x[j], sum);
                v[j] = br * da;
            }
            st_tile_f16(tile(U_DS), r, c0, v);  // dG over dS
        }
        sPart[(2 * s + me.cg) * HB + r] = sum;
        // dk = dK + dS^T Q + dN^T W (column half s)
        me.ld(tbase, UC_DK, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += xk[j];
        if (valid) st_global(dk + grow * DH + 64 * s + c0, v);
    }
    sync_operands();
    if (ok && tid < HB && prow0 + tid < L)
        dbeta[(long long)hd * L + prow0 + tid] =
            sPart[tid] + sPart[HB + tid] + sPart[2 * HB + tid] + sPart[3 * HB + tid];

    // ---- B4: dw = D dR_w + (dM^T Q + dN K + dG W + dG^T W) - (U dK + What dP^T)
    ISSUE(for (int c = 0; c < 2; ++c) {
        const uint32_t wc = ta(U_W + 2 * c);
        mma64(dst(tbase, c, UC_W1), ta(U_M), A_T, ta(U_Q + c), B_N, 1, TILE, false);
        mma64(dst(tbase, c, UC_W1), ta(U_X), A_N, ta(U_W + 2 * c + 1), B_N, 1, TILE, true);
        mma64(dst(tbase, c, UC_W1), ta(U_DS), A_N, wc, B_N, 1, TILE, true);
        mma64(dst(tbase, c, UC_W1), ta(U_DS), A_T, wc, B_N, 1, TILE, true);
        mma64(dst(tbase, c, UC_W2), ta(U_U), A_N, ta(U_DK + c), B_N, 1, TILE, false);
        for (int k = 0; k < 2; ++k)
            mma64(dst(tbase, c, UC_W2), ta(U_WH + k), A_N, ta(U_DP + 2 * c + k), B_T, 1, TILE, true);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, UC_W1, v);
        me.ld(tbase, UC_W2, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] -= x[j];
        me.ld(tbase, UC_DRW, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = fmaf(br, x[j], v[j]);
        if (valid) st_global(dw + grow * DH + 64 * s + c0, v);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 25);
    if (warp == 0) tmem_dealloc(tbase, 512);
}

#undef ISSUE

template <typename TO>
cudaError_t launch_adj(const CUtensorMap *m, const PrepDims &Dm, const PrepInputs &in,
                       const PrepGrads &g, const int *saved, int *err, cudaStream_t st)
{
    auto k = ut_adj128_kernel<TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, U_SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(2 * Dm.nblk, Dm.nh), NT, U_SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], in.beta,
                                                     Dm.L, Dm.nblk, g.dQt, g.dKt, g.dSd,
                                                     static_cast<TO *>(g.dq), static_cast<TO *>(g.dk),
                                                     static_cast<TO *>(g.dw), g.dbeta, saved, err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

cudaError_t prep_backward_ut128(const PrepDims &Dm, const PrepInputs &in, const PrepGrads &g,
                                const UtSave &sv, const int *saved, int *err, cudaStream_t st)
{
    if (!prep_forward_ut128_supported(Dm, in) || (long long)Dm.nh * Dm.nblk * 2 * DH >= (1LL << 31))
        return cudaErrorInvalidValue;
    const uint64_t nb = (uint64_t)Dm.nh * Dm.nblk;
    CUtensorMap ca[4];
    if (!make_map_2d(&ca[0], sv.Kta, F16, DH, nb * HB, HB) || !make_map_2d(&ca[1], sv.Qtb, F16, DH, nb * HB, HB) ||
        !make_map_2d(&ca[2], sv.Pa, F16, DH, nb * DH, HB) || !make_map_2d(&ca[3], sv.Pb, F16, DH, nb * DH, HB))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(compose_adj128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CA_SMEM);
    if (e != cudaSuccess) return e;
    compose_adj128_kernel<<<dim3(Dm.nblk, Dm.nh), NT, CA_SMEM, st>>>(
        ca[0], ca[1], ca[2], ca[3], Dm.nblk, const_cast<float *>(g.dQt), const_cast<float *>(g.dKt), g.dPm,
        g.dSd, sv.dP, saved, err);
    count_launches();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap m[8];
    if (!make_map_3d(&m[0], in.w, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[1], in.q, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&m[2], in.k, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_2d(&m[3], sv.What, F16, DH, nb * 2 * HB, HB) ||
        !make_map_2d(&m[4], sv.U, F16, HB, nb * 2 * HB, HB) || !make_map_2d(&m[5], sv.X, F16, HB, nb * 2 * HB, HB) ||
        !make_map_2d(&m[6], sv.M, F16, HB, nb * 2 * HB, HB) ||
        !make_map_2d(&m[7], sv.dP, F16, DH, nb * 2 * DH, HB))
        return cudaErrorInvalidValue;
    if (Dm.odt == F32) return launch_adj<float>(m, Dm, in, g, saved, err, st);
    return launch_adj<bf16>(m, Dm, in, g, saved, err, st);
}

}  // namespace path
