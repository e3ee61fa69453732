// Forward UT prep of one 128-position block on 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory), head dim 64, bf16 inputs.
//
// Per 64-position half (positions s..e, H_t = I - beta_t w_t w_t^T), the UT
// transform in closed form (Paper-Notes "训练策略": T^{-1} = (I + strictLower(D W W^T))^{-1} D,
// and the full-matrix form of the block's logits):
//   A = strictLower(D W W^T), N = strictLower(W K^T), M = lower(Q W^T),
//   [What | U] = (I + A)^{-1} D [W | N]
//   Qtil = Q - M What, Ktil = K - U^T W, P = I - W^T What, Sd = lower(Q K^T - M U)
// and the 128-block from its halves a (first) and b:
//   Qtil[a] = Qtil_a, Qtil[b] = Qtil_b P_a, Ktil[a] = Ktil_a P_b^T, Ktil[b] = Ktil_b,
//   P = P_b P_a, Sd = [[Sd_aa, 0], [Qtil_b Ktil_a^T, Sd_bb]].
//
// The inverse (I + A)^{-1} is not reached by substitution. With E the block
// diagonal of I + A in 16 x 16 blocks (inverted on the CUDA cores) and
// N' = E^{-1} A_off (A_off: A outside those blocks), N' is strictly lower in
// 16-row blocks, so N'^4 = 0 and
//   (I + A)^{-1} = (I + N')^{-1} E^{-1} = (I + N'^2)(I - N') E^{-1}.
// Applied to D [W | N] that is three dependent products:
//   Z = E^{-1} D [W | N],  Z1 = Z - N' Z (with N'^2 = N' N'),  [What | U] = Z1 + N'^2 Z1.
// Every product is an M = 64 MMA on fp16 operands with fp32 accumulation (the
// bf16 inputs are exact in fp16); both halves run side by side (ut_tc.cuh).
//
// With a save area (a workspace sized for the backward) the kernel also writes
// what the adjoint (prep_bwd_ut.cu) reads instead of recomputing it: per half
// What, U, -M and X = (I + A)^{-1} (the same factors applied to the identity:
// Z1x = (I - N') E^{-1}, X = (I + N'^2) Z1x), and the composition's inputs
// Ktil_a, Qtil_b, P_a, P_b, all fp16 as the products read them, by TMA stores
// of the operand tiles.
#include "prep.cuh"
#include "runtime.cuh"
#include "ut_tc.cuh"

namespace path {

namespace {

using namespace tc;
using namespace uttc;

constexpr int NT = 256;

// shared-memory tiles (8 KB each)
enum {
    T_WA = 0, T_KA = 1, T_WB = 2, T_KB = 3,  // W_h, K_h adjacent: [W_h; K_h] is one 128-row B
    T_QA = 4, T_QB = 5,
    T_DA = 6, T_DB = 7,    // E^{-1}, then N'^2
    T_F1 = 8,              // per half (b at +3): A_off, D W, D N (B of the first product)
    T_MA = 14, T_MB = 15,  // -M
    T_NA = 16, T_NB = 17,  // -N'
    T_Z = 18,              // per half (b at +2): [Zw, Zn] = Z, then Z1, then [What, U]
    NTILES = 22,
    // composition operands (over the T_F1 tiles, free by then)
    T_KTA = 8, T_QTB = 9, T_PA = 10, T_PB = 11,
};
constexpr int SA16_OFF = NTILES * TILE;              // [2][4][16][16] fp32 diagonal blocks of A
constexpr int BETA_OFF = SA16_OFF + 2 * 4 * 256 * 4;  // [128] beta
constexpr int BAR_OFF = BETA_OFF + 128 * 4;
constexpr int SMEM = BAR_OFF + 64 + 1024;             // + 1024-byte alignment slack

// tensor-memory columns
constexpr int C_G = 0, C_N = 64, C_M = 128, C_S = 192;  // W W^T, W K^T, Q W^T, Q K^T (then Sd)
constexpr int C_Z = 256;                               // N' | Zw | Zn (then Z1, [What | U])
constexpr int C_N2 = 0, C_ZX = 64;                     // N'^2; saving: the X products
constexpr int C_QT = 64, C_KT = 128, C_P = 0;          // -M What, U^T W, W^T What
constexpr int C_C1 = 256, C_C2 = 320;                  // composition

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
// ([nh Lp, 64] fp16), Pm ([nh nblk 64, 64] fp16) in 64 x 64 tiles, Sd
// ([nh nblk 128, 128] fp32) in 64-row boxes of 32 columns.
template <bool SAVE>
__global__ void __launch_bounds__(NT, 1)
    prep_fwd_ut_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mQ,
                       const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mQt,
                       const __grid_constant__ CUtensorMap mKt, const __grid_constant__ CUtensorMap mPm,
                       const __grid_constant__ CUtensorMap mSd, const __grid_constant__ CUtensorMap mSvH,
                       const __grid_constant__ CUtensorMap mSvB, const float *beta, int L, int nblk,
                       int nsm, int *err)
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
        mbar_expect_tx(&bars[0], 6 * TILE);
        for (int h = 0; h < 2; ++h) {
            const int y = J * BT + h * HB;
            tma_load_3d(tile(h ? T_WB : T_WA), &mW, 0, y, hd, &bars[0]);
            tma_load_3d(tile(h ? T_KB : T_KA), &mK, 0, y, hd, &bars[0]);
            tma_load_3d(tile(h ? T_QB : T_QA), &mQ, 0, y, hd, &bars[0]);
        }
        // one CTA per SM, started in grid order: the block nsm places further on
        // starts on an SM this wave frees; its inputs go to L2 meanwhile
        const long long n2 = (long long)hd * nblk + J + nsm;
        if (n2 < (long long)nblk * gridDim.y) {
            const int J2 = (int)(n2 % nblk), h2 = (int)(n2 / nblk);
            for (int h = 0; h < 2; ++h) {
                tma_prefetch_3d(&mW, 0, J2 * BT + h * HB, h2);
                tma_prefetch_3d(&mK, 0, J2 * BT + h * HB, h2);
                tma_prefetch_3d(&mQ, 0, J2 * BT + h * HB, h2);
            }
        }
    }
    if (warp == 0) tmem_alloc(tslot, 512);
    // the E^{-1} tiles: only their diagonal blocks are written below
    for (int i = tid; i < 2 * (int)TILE / 16; i += NT)
        reinterpret_cast<uint4 *>(tile(T_DA))[i] = make_uint4(0u, 0u, 0u, 0u);
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
    const int blk = hd * nblk + J;
    // the save maps: mSvH over What, U, X, -M ([nb 2 64, 64] each, stacked at
    // hstride rows), mSvB over Kta, Qtb, Pa, Pb ([nb 64, 64] each, bstride rows)
    const int hstride = nblk * gridDim.y * 2 * HB, bstride = nblk * gridDim.y * HB;
    constexpr int T_ZX = 12;  // + h: Z1x (over F1 tiles, free from level 1 to 4)
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

    // ---- level 0: [W; Q] [W; K]^T per half (bf16 operands)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const uint32_t wk = ta(hh ? T_WB : T_WA);
        mma64(dst(tbase, hh, C_G), wk, A_N, wk, B_T, 2, TILE, false, AB_BF16);
        mma64(dst(tbase, hh, C_M), ta(hh ? T_QB : T_QA), A_N, wk, B_T, 2, TILE, false, AB_BF16);
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
        st_tile_f16(tile(T_F1 + 3 * h), r, c0, x);
        me.ld(tbase, C_N, v);  // D N, N = strictLower(W K^T)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j < r ? br * v[j] : 0.f;
        st_tile_f16(tile(T_F1 + 3 * h + 2), r, c0, v);
        me.ld(tbase, C_M, v);  // -M, M = lower(Q W^T)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = c0 + j <= r ? -v[j] : 0.f;
        st_tile_f16(tile(h ? T_MB : T_MA), r, c0, v);
        // W to fp16 in place (an operand beside fp16 intermediates from here on), and D W
        uint8_t *tw = tile(h ? T_WB : T_WA);
        ld_tile_bf16(tw, r, c0, v);
        st_tile_f16(tw, r, c0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= br;
        st_tile_f16(tile(T_F1 + 3 * h + 1), r, c0, v);
    }
    sync_operands();
    if (SAVE && ok && storer) {  // -M of both halves
        for (int hh = 0; hh < 2; ++hh) tma_store_2d(&mSvH, 0, 3 * hstride + (blk * 2 + hh) * HB, tile(T_MA + hh));
        bulk_commit();
    }
    if (ok) {
        uint8_t *const dinv[2] = {tile(T_DA), tile(T_DB)};
        diag_block_inverses(sA16, dinv);
    }
    sync_operands();

    // ---- level 1: [N' | Zw | Zn] = E^{-1} [A_off | D W | D N]
    ISSUE(for (int hh = 0; hh < 2; ++hh)
              mma64(dst(tbase, hh, C_Z), ta(T_DA + hh), A_N, ta(T_F1 + 3 * hh), B_N, 3, TILE, false));
    wait_mma();
    if (ok) {
        me.ld(tbase, C_Z, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        st_tile_f16(tile(T_NA + h), r, c0, v);
        me.ld(tbase, C_Z + 64, v);
        st_tile_f16(tile(T_Z + 2 * h), r, c0, v);
        me.ld(tbase, C_Z + 128, v);
        st_tile_f16(tile(T_Z + 2 * h + 1), r, c0, v);
    }
    sync_operands();

    // ---- level 2: Z1 = Z + (-N') Z (in place in tensor memory), N'^2 = (-N')(-N');
    // saving: (-N') E^{-1}, so that Z1x = E^{-1} + (-N') E^{-1}
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        mma64(dst(tbase, hh, C_Z + 64), ta(T_NA + hh), A_N, ta(T_Z + 2 * hh), B_N, 2, TILE, true);
        mma64(dst(tbase, hh, C_N2), ta(T_NA + hh), A_N, ta(T_NA + hh), B_N, 1, TILE, false);
        if (SAVE) mma64(dst(tbase, hh, C_ZX), ta(T_NA + hh), A_N, ta(T_DA + hh), B_N, 1, TILE, false);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, C_Z + 64, v);
        st_tile_f16(tile(T_Z + 2 * h), r, c0, v);
        me.ld(tbase, C_Z + 128, v);
        st_tile_f16(tile(T_Z + 2 * h + 1), r, c0, v);
        if (SAVE) {  // E^{-1} read before N'^2 replaces it
            me.ld(tbase, C_ZX, v);
            ld_tile_f16(tile(T_DA + h), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += x[j];
            st_tile_f16(tile(T_ZX + h), r, c0, v);
        }
        me.ld(tbase, C_N2, v);
        st_tile_f16(tile(T_DA + h), r, c0, v);
    }
    sync_operands();

    // ---- level 3: [What | U] = Z1 + N'^2 Z1; saving: N'^2 Z1x (X = Z1x + N'^2 Z1x)
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        mma64(dst(tbase, hh, C_Z + 64), ta(T_DA + hh), A_N, ta(T_Z + 2 * hh), B_N, 2, TILE, true);
        if (SAVE) mma64(dst(tbase, hh, C_ZX), ta(T_DA + hh), A_N, ta(T_ZX + hh), B_N, 1, TILE, false);
    });
    wait_mma();
    if (ok) {
        me.ld(tbase, C_Z + 64, v);
        st_tile_f16(tile(T_Z + 2 * h), r, c0, v);
        me.ld(tbase, C_Z + 128, v);
        st_tile_f16(tile(T_Z + 2 * h + 1), r, c0, v);
        if (SAVE) {  // X over -N' (read by no product since level 2)
            me.ld(tbase, C_ZX, v);
            ld_tile_f16(tile(T_ZX + h), r, c0, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += x[j];
            st_tile_f16(tile(T_NA + h), r, c0, v);
        }
    }
    // the -M tiles become staging in level 4's epilogue: their save is read by now
    if (SAVE && storer) bulk_wait_read<0>();
    sync_operands();
    if (SAVE && ok && storer) {
        for (int hh = 0; hh < 2; ++hh) {
            const int y = (blk * 2 + hh) * HB;
            tma_store_2d(&mSvH, 0, y, tile(T_Z + 2 * hh));                 // What
            tma_store_2d(&mSvH, 0, hstride + y, tile(T_Z + 2 * hh + 1));   // U
            tma_store_2d(&mSvH, 0, 2 * hstride + y, tile(T_NA + hh));      // X
        }
        bulk_commit();
    }

    // ---- level 4: -M What, Q K^T - M U, U^T W, W^T What
    ISSUE(for (int hh = 0; hh < 2; ++hh) {
        const uint32_t wh = ta(T_Z + 2 * hh), u = ta(T_Z + 2 * hh + 1), w = ta(hh ? T_WB : T_WA);
        mma64(dst(tbase, hh, C_QT), ta(T_MA + hh), A_N, wh, B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_S), ta(T_MA + hh), A_N, u, B_N, 1, TILE, true);
        mma64(dst(tbase, hh, C_KT), u, A_T, w, B_N, 1, TILE, false);
        mma64(dst(tbase, hh, C_P), w, A_T, wh, B_N, 1, TILE, false);
    });
    wait_mma();
    // staging: tiles free by now (F4's and the composition's, kept apart so the
    // first stores can still be reading theirs while the second are written)
    enum { S_QA = 12, S_KB = 13, S_SDA = 6, S_SDB = 14, S_KA = 0, S_QB = 1, S_PM = 2, S_SDBA = 3 };
    const int brow = hd * Lp + J * BT;            // block's first row in [nh Lp] (fits int32)
    const int sdrow = (hd * nblk + J) * BT;       // and in [nh nblk 128]
    if (ok) {
        // Qtil_h = Q - M What
        me.ld(tbase, C_QT, v);
        ld_tile_bf16(tile(h ? T_QB : T_QA), r, c0, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += x[j];
        st_tile_f16(tile(h ? T_QTB : S_QA), r, c0, v);
        // Ktil_h = K - U^T W
        me.ld(tbase, C_KT, v);
        ld_tile_bf16(tile(h ? T_KB : T_KA), r, c0, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = x[j] - v[j];
        st_tile_f16(tile(h ? S_KB : T_KTA), r, c0, v);
        // P_h = I - W^T What
        me.ld(tbase, C_P, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (c0 + j == r ? 1.f : 0.f) - v[j];
        st_tile_f16(tile(h ? T_PB : T_PA), r, c0, v);
        // Sd_hh = lower(Q K^T - M U) (the block above the diagonal blocks is never
        // read: the attention kernels mask it)
        me.ld(tbase, C_S, v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (c0 + j > r) v[j] = 0.f;
        st_box_f32(tile((h ? S_SDB : S_SDA) + me.cg), r, v);
    }
    sync_operands();

    // ---- level 5: the 128-block from its halves; meanwhile Qtil[a], Ktil[b], Sd_aa, Sd_bb go out
    ISSUE({
        mma64(dst(tbase, 0, C_C1), ta(T_KTA), A_N, ta(T_PB), B_T, 1, TILE, false);  // Ktil_a P_b^T
        mma64(dst(tbase, 0, C_C2), ta(T_PB), A_N, ta(T_PA), B_N, 1, TILE, false);   // P_b P_a
        mma64(dst(tbase, 1, C_C1), ta(T_QTB), A_N, ta(T_PA), B_N, 1, TILE, false);  // Qtil_b P_a
        mma64(dst(tbase, 1, C_C2), ta(T_QTB), A_N, ta(T_KTA), B_T, 1, TILE, false); // Qtil_b Ktil_a^T
    });
    if (ok && storer) {
        if (SAVE)  // the composition's inputs: Ktil_a, Qtil_b, P_a, P_b
            for (int i = 0; i < 4; ++i) tma_store_2d(&mSvB, 0, i * bstride + blk * HB, tile(T_KTA + i));
        tma_store_2d(&mQt, 0, brow, tile(S_QA));
        tma_store_2d(&mKt, 0, brow + HB, tile(S_KB));
        for (int b = 0; b < 2; ++b) {
            tma_store_2d(&mSd, 32 * b, sdrow, tile(S_SDA + b));
            tma_store_2d(&mSd, HB + 32 * b, sdrow + HB, tile(S_SDB + b));
        }
        bulk_commit();
    }
    wait_mma();
    if (ok) {
        me.ld(tbase, C_C1, v);
        st_tile_f16(tile(h ? S_QB : S_KA), r, c0, v);  // Ktil[a] = Ktil_a P_b^T, Qtil[b] = Qtil_b P_a
        me.ld(tbase, C_C2, v);
        if (h == 0)
            st_tile_f16(tile(S_PM), r, c0, v);         // P = P_b P_a
        else
            st_box_f32(tile(S_SDBA + me.cg), r, v);    // Sd[b, a] = Qtil_b Ktil_a^T
    }
    sync_operands();
    if (ok && storer) {
        tma_store_2d(&mKt, 0, brow, tile(S_KA));
        tma_store_2d(&mQt, 0, brow + HB, tile(S_QB));
        tma_store_2d(&mPm, 0, (hd * nblk + J) * HB, tile(S_PM));
        for (int b = 0; b < 2; ++b) tma_store_2d(&mSd, 32 * b, sdrow + HB, tile(S_SDBA + b));
        bulk_commit();
    }
    if (storer) bulk_wait_all();  // the staging is read (and written out) before the CTA exits
#undef ISSUE
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!ok && tid == 0 && err) atomicCAS(err, 0, 21);
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace

bool prep_forward_ut_supported(const PrepDims &Dm, const PrepInputs &in)
{
    const uintptr_t al = reinterpret_cast<uintptr_t>(in.q) | reinterpret_cast<uintptr_t>(in.k) |
                         reinterpret_cast<uintptr_t>(in.w);
    // tile row coordinates of the output tensor maps are int32
    return Dm.d == HB && Dm.dt == BF16 && (al & 15u) == 0 &&
           (long long)Dm.nh * Dm.nblk * BT < (1LL << 31);
}

cudaError_t prep_forward_ut(const PrepDims &Dm, const PrepInputs &in, const PrepOutputs &out,
                            const UtSave *save, int *err, cudaStream_t st)
{
    if (!prep_forward_ut_supported(Dm, in)) return cudaErrorInvalidValue;
    CUtensorMap mW, mQ, mK, mQt, mKt, mPm, mSd;
    const uint64_t rows = (uint64_t)Dm.nh * Dm.nblk * BT;
    if (!make_map_3d(&mW, in.w, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&mQ, in.q, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_3d(&mK, in.k, BF16, HB, Dm.L, Dm.nh, HB) ||
        !make_map_2d(&mQt, out.Qt, F16, HB, rows, HB) || !make_map_2d(&mKt, out.Kt, F16, HB, rows, HB) ||
        !make_map_2d(&mPm, out.Pm, F16, HB, (uint64_t)Dm.nh * Dm.nblk * HB, HB) ||
        !make_map_f32_2d(&mSd, out.Sd, BT, rows, HB))
        return cudaErrorInvalidValue;
    CUtensorMap mSvH{}, mSvB{};  // unused without a save area
    if (save) {
        // What, U, X, M and Kta, Qtb, Pa, Pb lie back to back (carve_ut_save): one map each
        const uint64_t nb = (uint64_t)Dm.nh * Dm.nblk, hsz = nb * 2 * HB * HB, bsz = nb * HB * HB;
        if (save->U != save->What + hsz || save->X != save->U + hsz || save->M != save->X + hsz ||
            save->Qtb != save->Kta + bsz || save->Pa != save->Qtb + bsz || save->Pb != save->Pa + bsz ||
            nb * 4 * BT >= (1ull << 31))
            return cudaErrorInvalidValue;
        if (!make_map_2d(&mSvH, save->What, F16, HB, 4 * nb * 2 * HB, HB) ||
            !make_map_2d(&mSvB, save->Kta, F16, HB, 4 * nb * HB, HB))
            return cudaErrorInvalidValue;
    }
    auto k = save ? prep_fwd_ut_kernel<true> : prep_fwd_ut_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(Dm.nblk, Dm.nh), NT, SMEM, st>>>(mW, mQ, mK, mQt, mKt, mPm, mSd, mSvH, mSvB, in.beta, Dm.L,
                                              Dm.nblk, sm_count(), err);
    count_launches();
    return cudaGetLastError();
}

}  // namespace path
