// Forward UT prep of one 128-position block on 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory), head dim 128, bf16 inputs.
//
// The same closed form as the head-dim-64 kernel (prep_fwd_ut.cu), per
// 64-position half (Paper-Notes "训练策略": T^{-1} = (I + strictLower(D W W^T))^{-1} D):
//   A = strictLower(D W W^T), N = strictLower(W K^T), M = lower(Q W^T),
//   [What | U] = (I + A)^{-1} D [W | N]   (by the block-diagonal / nilpotent
//   factors E^{-1}, N', N'^2 of prep_fwd_ut.cu)
//   Qtil = Q - M What, Ktil = K - U^T W, P = I - W^T What, Sd = lower(Q K^T - M U)
// and the block from its halves a, b:
//   Qtil[a] = Qtil_a, Qtil[b] = Qtil_b P_a, Ktil[a] = Ktil_a P_b^T, Ktil[b] = Ktil_b,
//   P = P_b P_a, Sd = [[Sd_aa, 0], [Qtil_b Ktil_a^T, Sd_bb]]
// (gist.science section 3, "FlashAttention-Stijl Algoritme").
//
// At d = 128 every d-wide matrix of a half (W, K, Q, What, Qtil, Ktil: 64 x 128)
// is two 64-column tiles, and P_h, P (128 x 128) four. Position x position
// matrices (A, N', M, U: 64 x 64) are as at d = 64. Products are M = 64 MMAs
// on fp16 operands with fp32 accumulation, both halves side by side in tensor
// memory (ut_tc.cuh); a 128-row result (P_h, P) is two M = 64 row blocks. The
// four results of the halves' last level (M What, U^T W, W^T What in two row
// blocks, and M U added to Q K^T) exceed the 512 tensor-memory columns by one
// row block of P_h: that one is issued after the others have been read.
//
// With a save area (a workspace sized for the backward) the kernel also writes
// what the adjoint (prep_bwd_ut128.cu) reads instead of recomputing it: per
// half What, U, -M and X = (I + A)^{-1} (the same three factors applied to the
// identity: Z1x = (I - N') E^{-1}, X = (I + N'^2) Z1x), and the composition's
// inputs Ktil_a, Qtil_b, P_a, P_b, all fp16 as the products read them (What, U,
// X and -M by TMA stores of the operand tiles).
#include "prep.cuh"
#include "runtime.cuh"
#include "ut_tc.cuh"

namespace path {

namespace {

using namespace tc;
using namespace uttc;

constexpr int NT = 256;
constexpr int DH = 128;  // head dim

// shared-memory tiles (8 KB: 64 x 64 16-bit, or a 64-row x 32-column fp32 box)
__host__ __device__ constexpr int T_W(int h, int c) { return 4 * h + 2 * c; }      // W_h, columns 64c..
__host__ __device__ constexpr int T_K(int h, int c) { return 4 * h + 2 * c + 1; }  // K_h (after W_h: [W; K] is one 128-row B)
__host__ __device__ constexpr int T_Q(int h, int c) { return 8 + 2 * h + c; }
constexpr int T_E = 12;   // + h: E^{-1}_h, then N'^2_h
constexpr int T_M = 14;   // + h: -M_h; then the fp32 boxes of Sd_aa (14, 15) and Sd_bb (16, 17)
constexpr int T_NN = 16;  // + h: -N'_h
constexpr int T_F = 18;   // + 4h: [A_off | D W (2) | D N], then Z = [Zw (2) | Zn] -> [What | U];
                          // then P_a (18 + 2 rk + ck) and P_b (22 + 2 ck + rb); then P's staging
constexpr int NTILES = 26;
constexpr int SA16_OFF = NTILES * TILE;               // [2][4][16][16] fp32 diagonal blocks of A
constexpr int BETA_OFF = SA16_OFF + 2 * 4 * 256 * 4;  // [128] beta
constexpr int BAR_OFF = BETA_OFF + 128 * 4;
constexpr int SMEM = BAR_OFF + 64 + 1024;             // + 1024-byte alignment slack
static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");

// tensor-memory columns (both halves share them: lane offsets 0 / 16)
constexpr int C_G = 0, C_N = 64, C_M = 128, C_S = 192;  // W W^T, W K^T, Q W^T, Q K^T (then Sd)
constexpr int C_Z = 256;                                // N' | Zw (2) | Zn, then Z1, [What | U]
constexpr int C_N2 = 0, C_ZX = 64;                      // N'^2; saving: the X products
constexpr int C_QT = 0, C_KT = 256, C_P0 = 384;         // -M What, U^T W, rows 0..63 of W^T What
constexpr int C_P1 = 0;                                 // rows 64..127 of W^T What
constexpr int C_C1 = 0, C_C2 = 128, C_C3 = 256;         // composition

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Row r of a 64-row fp32 TMA box of 32 columns (128-byte rows, 128-byte swizzle).
__device__ __forceinline__ void st_box_f32(uint8_t *box, int r, const float (&v)[32])
{
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float4 *>(box + r * 128 + ((k ^ (r & 7)) << 4)) =
            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}

// Outputs leave through shared-memory staging and TMA tensor stores: Qt, Kt
// ([nh Lp, 128] fp16) and Pm ([nh nblk 128, 128] fp16) in 64 x 64 tiles, Sd
// ([nh nblk 128, 128] fp32) in 64-row boxes of 32 columns.
template <bool SAVE>
__global__ void __launch_bounds__(NT, 1)
    prep_fwd_ut128_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mQ,
                          const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mQt,
                          const __grid_constant__ CUtensorMap mKt, const __grid_constant__ CUtensorMap mPm,
                          const __grid_constant__ CUtensorMap mSd, const __grid_constant__ CUtensorMap mSvW,
                          const __grid_constant__ CUtensorMap mSvH, const float *beta, int L, int nblk,
                          int nsm, UtSave sv, int *err)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    auto tile = [&](int i) { return sm + i * TILE; };
    const uint32_t s0 = smem_u32(sm);
    auto ta = [&](int i) { return s0 + (uint32_t)i * TILE; };
    float *sA16 = reinterpret_cast<float *>(sm + SA16_OFF);
    float *sB = reinterpret_cast<float *>(sm + BETA_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + BAR_OFF);  // [0] loads, [1] MMA
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int J = blockIdx.x, hd = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Lp = nblk * BT;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        // rows past L read as zero (w = 0, beta = 0: H = I there)
        mbar_expect_tx(&bars[0], 12 * TILE);
        for (int h = 0; h < 2; ++h) {
            const int y = J * BT + h * HB;
            for (int c = 0; c < 2; ++c) {
                tma_load_3d(tile(T_W(h, c)), &mW, 64 * c, y, hd, &bars[0]);
                tma_load_3d(tile(T_K(h, c)), &mK, 64 * c, y, hd, &bars[0]);
                tma_load_3d(tile(T_Q(h, c)), &mQ, 64 * c, y, hd, &bars[0]);
            }
        }
        // one CTA per SM, started in grid order: the block nsm places further on
        // starts on an SM this wave frees; its inputs go to L2 meanwhile
        const long long n2 = (long long)hd * nblk + J + nsm;
        if (n2 < (long long)nblk * gridDim.y) {
            const int J2 = (int)(n2 % nblk), h2 = (int)(n2 / nblk);
            for (int h = 0; h < 2; ++h)
                for (int c = 0; c < 2; ++c) {
                    tma_prefetch_3d(&mW, 64 * c, J2 * BT + h * HB, h2);
                    tma_prefetch_3d(&mK, 64 * c, J2 * BT + h * HB, h2);
                    tma_prefetch_3d(&mQ, 64 * c, J2 * BT + h * HB, h2);
                }
        }
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    // the E^{-1} tiles: only their diagonal blocks are written below
    for (int i = tid; i < 2 * (int)TILE / 16; i += NT)
        reinterpret_cast<uint4 *>(tile(T_E))[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tid < BT) {
        const int p = J * BT + tid;
        sB[tid] = p < L ? beta[(long long)hd * L + p] : 0.f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tslot;
    bool ok = mbar_wait(&bars[0], 0, WAIT_LIMIT_NS);
    ok = __syncthreads_and(ok);

    const Me me;
    const int h = me.h, r = me.r, c0 = 32 * me.cg;
    const float br = sB[h * HB + r];
    const int F = T_F + 4 * h;  // this half's F / Z tiles
    const long long blk = (long long)hd * nblk + J;
    // the save maps: mSvW over What ([nb 2 64, 128]), mSvH over U, X, -M ([nb 2 64, 64]
    // each, stacked at hs rows); a half's rows start at hy
    const int hs = nblk * gridDim.y * 2 * HB;
    const bool storer = tid == 32;  // issues every TMA store (and waits for its own groups)
    uint32_t phase = 0;
    // one level: operands written and fenced, barrier; one thread issues the
    // products and commits; everyone waits for them
    auto sync_operands = [&]() {
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok);
    };
    auto wait_mma = [&]() {
        if (ok && !mbar_wait(&bars[1], phase, WAIT_LIMIT_NS)) ok = false;
        phase ^= 1;
        fence_after_sync();
    };
#define ISSUE(...)                                \
    do {                                          \
        if (ok && warp == 0) {                    \
            fence_after_sync();                   \
            if (lane == 0) {                      \
                __VA_ARGS__;                      \
                commit(&bars[1]);                 \
            }                                     \
            __syncwarp();                         \
        }                                         \
    } while (0)

    float v[32], x[32];

    // ---- level 0: [W; Q] [W; K]^T per half over both 64-column chunks (bf16 operands)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        for (int c = 0; c < 2; ++c) {
            const uint32_t wk = ta(T_W(hh, c));
            mma64(dst(tbase, hh, C_G), wk, A_N, wk, B_T, 2, TILE, c > 0, AB_BF16);
            mma64(dst(tbase, hh, C_M), ta(T_Q(hh, c)), A_N, wk, B_T, 2, TILE, c > 0, AB_BF16);
        }
    });
    wait_mma();
    if (ok) {
        // A = strictLower(D W W^T): diagonal 16-blocks to sA16 (fp32), the rest to A_off
        me.ld(tbase, C_G, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int col = c0 + j;
            const float a = col < r ? br * v[j] : 0.f;
            if ((col >> 4) == (r >> 4)) {
                sA16[((h * 4 + (r >> 4)) * 16 + (r & 15)) * 16 + (col & 15)] = a;
                x[j] = 0.f;
            } else {
                x[j] = a;
            }
        }
        st_tile_f16(tile(F), r, c0, x);
        me.ld(tbase, C_N, v);  // D N, N = strictLower(W K^T)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j < r ? br * v[j] : 0.f;
        st_tile_f16(tile(F + 3), r, c0, v);
        me.ld(tbase, C_M, v);  // -M, M = lower(Q W^T)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j <= r ? -v[j] : 0.f;
        st_tile_f16(tile(T_M + h), r, c0, v);
        // W to fp16 in place (an operand beside fp16 intermediates from here on), and D W
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            uint8_t *tw = tile(T_W(h, c));
            ld_tile_bf16(tw, r, c0, v);
            st_tile_f16(tw, r, c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= br;
            st_tile_f16(tile(F + 1 + c), r, c0, v);
        }
    }
    sync_operands();
    if (SAVE && ok && storer) {  // -M of both halves
        for (int hh = 0; hh < 2; ++hh) tma_store_2d(&mSvH, 0, 2 * hs + (int)(blk * 2 + hh) * HB, tile(T_M + hh));
        bulk_commit();
    }
    if (ok) {
        uint8_t *const dinv[2] = {tile(T_E), tile(T_E + 1)};
        diag_block_inverses(sA16, dinv);
    }
    sync_operands();

    // ---- level 1: [N' | Zw | Zn] = E^{-1} [A_off | D W | D N]  (N = 256)
    ISSUE(for (int hh = 0; hh < 2; ++hh)
              mma64(dst(tbase, hh, C_Z), ta(T_E + hh), A_N, ta(T_F + 4 * hh), B_N, 4, TILE, false));
    wait_mma();
    if (ok) {
        me.ld(tbase, C_Z, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(T_NN + h), r, c0, v);
        // Z over the F tiles (their products are complete)
#pragma unroll 1
        for (int m = 0; m < 3; ++m) {
            me.ld(tbase, C_Z + 64 + 64 * m, v);
            st_tile_f16(tile(F + m), r, c0, v);
        }
    }
    sync_operands();

    // ---- level 2: Z1 = Z + (-N') Z (in place in tensor memory), N'^2 = (-N')(-N');
    // saving: (-N') E^{-1}, so that Z1x = E^{-1} + (-N') E^{-1}
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        mma64(dst(tbase, hh, C_Z + 64), ta(T_NN + hh), A_N, ta(T_F + 4 * hh), B_N, 3, TILE, true);
        mma64(dst(tbase, hh, C_N2), ta(T_NN + hh), A_N, ta(T_NN + hh), B_N, 1, TILE, false);
        if (SAVE) mma64(dst(tbase, hh, C_ZX), ta(T_NN + hh), A_N, ta(T_E + hh), B_N, 1, TILE, false);
    });
    wait_mma();
    if (ok) {
#pragma unroll 1
        for (int m = 0; m < 3; ++m) {
            me.ld(tbase, C_Z + 64 + 64 * m, v);
            st_tile_f16(tile(F + m), r, c0, v);
        }
        if (SAVE) {  // Z1x over the D N tile (read by level 1); E^{-1} read before N'^2 replaces it
            me.ld(tbase, C_ZX, v);
            ld_tile_f16(tile(T_E + h), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += x[j];
            st_tile_f16(tile(F + 3), r, c0, v);
        }
        me.ld(tbase, C_N2, v);
        st_tile_f16(tile(T_E + h), r, c0, v);
    }
    sync_operands();

    // ---- level 3: [What | U] = Z1 + N'^2 Z1; saving: N'^2 Z1x (X = Z1x + N'^2 Z1x)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        mma64(dst(tbase, hh, C_Z + 64), ta(T_E + hh), A_N, ta(T_F + 4 * hh), B_N, 3, TILE, true);
        if (SAVE) mma64(dst(tbase, hh, C_ZX), ta(T_E + hh), A_N, ta(T_F + 4 * hh + 3), B_N, 1, TILE, false);
    });
    wait_mma();
    if (ok) {
#pragma unroll 1
        for (int m = 0; m < 3; ++m) {
            me.ld(tbase, C_Z + 64 + 64 * m, v);
            st_tile_f16(tile(F + m), r, c0, v);
        }
        if (SAVE) {  // X over Z1x
            me.ld(tbase, C_ZX, v);
            ld_tile_f16(tile(F + 3), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += x[j];
            st_tile_f16(tile(F + 3), r, c0, v);
        }
    }
    // the -M tiles become staging in level 4's epilogue: their save is read by now
    if (SAVE && storer) bulk_wait_read<0>();
    sync_operands();
    if (SAVE && ok && storer) {  // What, U, X of both halves
        for (int hh = 0; hh < 2; ++hh) {
            const int f = T_F + 4 * hh, hy = (int)(blk * 2 + hh) * HB;
            tma_store_2d(&mSvW, 0, hy, tile(f));
            tma_store_2d(&mSvW, 64, hy, tile(f + 1));
            tma_store_2d(&mSvH, 0, hy, tile(f + 2));
            tma_store_2d(&mSvH, 0, hs + hy, tile(f + 3));
        }
        bulk_commit();
    }

    // ---- level 4: -M What, Q K^T - M U, U^T W, rows 0..63 of W^T What
    // (What_h: tiles F, F + 1; U_h: F + 2; W_h's two column tiles 2 TILE apart)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const int f = T_F + 4 * hh;
        mma64(dst(tbase, hh, C_QT), ta(T_M + hh), A_N, ta(f), B_N, 2, TILE, false);
        mma64(dst(tbase, hh, C_S), ta(T_M + hh), A_N, ta(f + 2), B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_KT), ta(f + 2), A_T, ta(T_W(hh, 0)), B_N, 2, 2 * TILE, false);
        mma64(dst(tbase, hh, C_P0), ta(T_W(hh, 0)), A_T, ta(f), B_N, 2, TILE, false);
    });
    wait_mma();
    const int brow = hd * Lp + J * BT;       // block's first row in [nh Lp] (fits int32)
    const int sdrow = (hd * nblk + J) * BT;  // and in [nh nblk 128]
    if (ok) {
        // Qtil_h = Q - M What, over Q_h in place (fp16)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            me.ld(tbase, C_QT + 64 * c, v);
            ld_tile_bf16(tile(T_Q(h, c)), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += x[j];
            st_tile_f16(tile(T_Q(h, c)), r, c0, v);
            if (SAVE && h == 1) st_global(sv.Qtb + (blk * HB + r) * DH + 64 * c + c0, v);
        }
        // Ktil_h = K - U^T W, over K_h in place (fp16)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            me.ld(tbase, C_KT + 64 * c, v);
            ld_tile_bf16(tile(T_K(h, c)), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = x[j] - v[j];
            st_tile_f16(tile(T_K(h, c)), r, c0, v);
            if (SAVE && h == 0) st_global(sv.Kta + (blk * HB + r) * DH + 64 * c + c0, v);
        }
        // Sd_hh = lower(Q K^T - M U) (the block above the diagonal blocks is never
        // read: the attention kernels mask it), over the -M and -N' tiles
        me.ld(tbase, C_S, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (c0 + j > r) v[j] = 0.f;
        st_box_f32(tile(T_M + 2 * h + me.cg), r, v);
    }
    // P_h goes over the What / U / X tiles in level 4b's epilogue: their save is read by now
    if (SAVE && storer) bulk_wait_read<0>();
    sync_operands();

    // ---- level 4b: rows 64..127 of W^T What, over the (read) -M What columns;
    // meanwhile Qtil[a], Ktil[b], Sd_aa, Sd_bb go out
    ISSUE(for (int hh = 0; hh < 2; ++hh)
              mma64(dst(tbase, hh, C_P1), ta(T_W(hh, 1)), A_T, ta(T_F + 4 * hh), B_N, 2, TILE, false));
    if (ok && storer) {
        for (int c = 0; c < 2; ++c) {
            tma_store_2d(&mQt, 64 * c, brow, tile(T_Q(0, c)));
            tma_store_2d(&mKt, 64 * c, brow + HB, tile(T_K(1, c)));
            tma_store_2d(&mSd, 32 * c, sdrow, tile(T_M + c));
            tma_store_2d(&mSd, HB + 32 * c, sdrow + HB, tile(T_M + 2 + c));
        }
        bulk_commit();
    }
    wait_mma();
    if (ok) {
        // P_h = I - W^T What (row i = 64 rb + r, column 64 ck + c0 + j): P_a in
        // tiles 18 + 2 rb + ck (K-chunks of the B operand by rows), P_b in tiles
        // 22 + 2 ck + rb (its two row blocks adjacent: a 128-row K-major B)
#pragma unroll 1
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll 1
            for (int ck = 0; ck < 2; ++ck) {
                me.ld(tbase, (rb ? C_P1 : C_P0) + 64 * ck, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = (64 * rb + r == 64 * ck + c0 + j ? 1.f : 0.f) - v[j];
                st_tile_f16(tile(h ? T_F + 4 + 2 * ck + rb : T_F + 2 * rb + ck), r, c0, v);
                if (SAVE) st_global((h ? sv.Pb : sv.Pa) + (blk * DH + 64 * rb + r) * DH + 64 * ck + c0, v);
            }
    }
    sync_operands();

    // ---- level 5: the 128-block from its halves
    ISSUE({
        for (int k = 0; k < 2; ++k) {
            // Ktil[a] = Ktil_a P_b^T (half a's lanes)
            mma64(dst(tbase, 0, C_C1), ta(T_K(0, k)), A_N, ta(T_F + 4 + 2 * k), B_T, 2, TILE, k > 0);
            // Qtil[b] = Qtil_b P_a (half b's lanes)
            mma64(dst(tbase, 1, C_C1), ta(T_Q(1, k)), A_N, ta(T_F + 2 * k), B_N, 2, TILE, k > 0);
            // P = P_b P_a, row block rb in the lanes of "half" rb
            for (int rb = 0; rb < 2; ++rb)
                mma64(dst(tbase, rb, C_C2), ta(T_F + 4 + 2 * k + rb), A_N, ta(T_F + 2 * k), B_N, 2, TILE,
                      k > 0);
            // Sd[b, a] = Qtil_b Ktil_a^T (half b's lanes)
            mma64(dst(tbase, 1, C_C3), ta(T_Q(1, k)), A_N, ta(T_K(0, k)), B_T, 1, TILE, k > 0);
        }
    });
    wait_mma();
    if (ok) {
        // Ktil[a] over Ktil_a's tiles, Qtil[b] over Qtil_b's (their products are complete)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            me.ld(tbase, C_C1 + 64 * c, v);
            st_tile_f16(tile(h ? T_Q(1, c) : T_K(0, c)), r, c0, v);
        }
        // P = P_b P_a, row 64 h + r, over P_a's tiles (18 + 2 rb + ck)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            me.ld(tbase, C_C2 + 64 * c, v);
            st_tile_f16(tile(T_F + 2 * h + c), r, c0, v);
        }
        // Sd[b, a] over W_a's tiles (fp32 boxes; read by no product since level 4b)
        me.ld(tbase, C_C3, v);
        if (h == 1) st_box_f32(tile(T_W(0, me.cg)), r, v);
    }
    sync_operands();
    if (ok && storer) {
        for (int c = 0; c < 2; ++c) {
            tma_store_2d(&mKt, 64 * c, brow, tile(T_K(0, c)));
            tma_store_2d(&mQt, 64 * c, brow + HB, tile(T_Q(1, c)));
            for (int rb = 0; rb < 2; ++rb)
                tma_store_2d(&mPm, 64 * c, (hd * nblk + J) * DH + 64 * rb, tile(T_F + 2 * rb + c));
            tma_store_2d(&mSd, 32 * c, sdrow + HB, tile(T_W(0, c)));
        }
        bulk_commit();
    }
    if (storer) bulk_wait_all();  // the staging is read (and written out) before the CTA exits
#undef ISSUE
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 23);
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace

bool prep_forward_ut128_supported(const PrepDims &Dm, const PrepInputs &in)
{
    const uintptr_t al = reinterpret_cast<uintptr_t>(in.q) | reinterpret_cast<uintptr_t>(in.k) |
                         reinterpret_cast<uintptr_t>(in.w);
    // tile row coordinates of the output tensor maps are int32
    return Dm.d == DH && Dm.dt == BF16 && (al & 15u) == 0 &&
           (long long)Dm.nh * Dm.nblk * BT < (1LL << 31);
}

cudaError_t prep_forward_ut128(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out,
                               const UtSave *save, int *err, cudaStream_t st)
{
    if (!prep_forward_ut128_supported(Dm, in) || out.tdt != F16) return cudaErrorInvalidValue;
    CUtensorMap mW, mQ, mK, mQt, mKt, mPm, mSd;
    const uint64_t rows = (uint64_t)Dm.nh * Dm.nblk * BT;
    if (!make_map_3d(&mW, in.w, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&mQ, in.q, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&mK, in.k, BF16, DH, Dm.L, Dm.nh, HB) ||
        !make_map_2d(&mQt, out.Qt, F16, DH, rows, HB) || !make_map_2d(&mKt, out.Kt, F16, DH, rows, HB) ||
        !make_map_2d(&mPm, out.Pm, F16, DH, (uint64_t)Dm.nh * Dm.nblk * DH, HB) ||
        !make_map_f32_2d(&mSd, out.Sd, BT, rows, HB))
        return cudaErrorInvalidValue;
    CUtensorMap mSvW{}, mSvH{};  // unused without a save area
    if (save) {
        // U, X, M lie back to back (carve_ut_save): one map
        const uint64_t nb = (uint64_t)Dm.nh * Dm.nblk, hsz = nb * 2 * HB * HB;
        if (save->X != save->U + hsz || save->M != save->X + hsz || nb * 3 * BT >= (1ull << 31))
            return cudaErrorInvalidValue;
        if (!make_map_2d(&mSvW, save->What, F16, DH, nb * 2 * HB, HB) ||
            !make_map_2d(&mSvH, save->U, F16, HB, 3 * nb * 2 * HB, HB))
            return cudaErrorInvalidValue;
    }
    auto k = save ? prep_fwd_ut128_kernel<true> : prep_fwd_ut128_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(Dm.nblk, Dm.nh), NT, SMEM, st>>>(mW, mQ, mK, mQt, mKt, mPm, mSd, mSvW, mSvH, in.beta, Dm.L,
                                              Dm.nblk, sm_count(), save ? *save : UtSave{}, err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace path
