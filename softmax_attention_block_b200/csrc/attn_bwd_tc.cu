// PaTH attention backward on tensor cores (sm_100a), head dim 64.
//
// One CTA per (128-key tile J, head), walking the query tiles I = last..J+1,
// then the diagonal tile I = J. Keys are the CTA's rows: TMEM lane j is key j
// for S^T, dP^T, dV and the chain adjoint Abar. Per tile pair:
//   MMA 1:  S^T  = Khat_{J,I} Qtil_I^T          (fp16)
//           dP^T = V_J dO_I^T                    (bf16)
//   threads: P = exp(scale S + c_i - c_j - lse_i), dZ = P (dP - delta_i),
//            dS = scale dZ; P^T (bf16) into tensor memory over the S^T columns
//            already read, dS^T (fp16) to shared memory (two buffers);
//            [gate] row sums of dS by warp reduce-scatter, column sums per thread
//   MMA 2:  dV   += P^T dO_I                   (bf16, A = P^T from tensor memory)
//           dP_I += Abar_{I+1}^T Khat_{J,I}     (fp16; operand [Abar | Khat] so
//                   the M=128 form applies, top half kept)
//           Abar  = Abar_{I+1} P_I + dS^T Qtil_I           (fp16, fp32 in TMEM)
//           dQtil_I += dS Khat_{J,I}                       (fp16)
// Khat_{J,I+1} = Khat_{J,I} P_I^T, so Abar is the adjoint carried back along
// the key-side transport chain; after the pair (J+1, J) it is dKtil_J. dQtil is
// staged in the pair's spent dS^T buffer by the drain warps and accumulates
// across CTAs by TMA tensor reduce-add, and so does dP_I (through an 8 KB box); the gate's
// row sums by fp32 atomics. The diagonal tile takes its logits from the UT prep
// and writes dS to the prep's adjoint instead (dSd), which carries it to dQ,
// dK, dW, dbeta.
//
// Issue order of the MMA warp per pair: dV (reads this pair's P^T), the next
// pair's MMA 1 (overwrites S^T / P^T and dP^T: the tensor pipe runs one
// thread's MMAs in issue order), then the rest of MMA 2. So the softmax of the
// next pair runs while the rest of this pair's MMA 2 executes, and the drain of
// this pair's results runs under the softmax after it. The operand stage goes
// back to the producer when the MMAs that read it complete.
#include <type_traits>

#include "attn.cuh"
#include "attn_tc.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

constexpr int D = 64;
// warps 0-7: softmax (two warpgroups, one per 64-query half); 8-11: drain of
// MMA 2's results; 12: TMA producer; 13: MMA issue; 14-15: idle
constexpr int NT = 512;
constexpr int NEW = 256;                 // softmax threads
constexpr int NDR = 128;                 // drain threads
constexpr int W_DRAIN0 = 8, W_PROD = 12, W_MMA = 13;
constexpr float LOG2E = 1.4426950408889634f;

struct BCfg {
    static constexpr int TILE = 128 * D * 2;     // 16 KB
    static constexpr int AB_OFF = 0;             // Abar operand (fp16), before the stages
    static constexpr int V_OFF = AB_OFF + TILE;
    // dS^T [keys x queries] fp16, 2 panels of 64 queries; two buffers (pairs it % 2),
    // each the fp32 staging of that pair's dQtil once MMA 2 has read it
    static constexpr int DS_BYTES = 2 * 16384;
    static constexpr int DS_OFF = V_OFF + TILE;
    static constexpr int ST_OFF = DS_OFF + 2 * DS_BYTES;
    // stage: Khat, Qtil, dO, P_I (8 KB), rows (lse, delta, c: 3 x 512 B)
    static constexpr int S_KH = 0, S_Q = TILE, S_DO = 2 * TILE, S_P = 3 * TILE, S_ROW = 3 * TILE + 8192;
    static constexpr int ST_BYTES = 3 * TILE + 8192 + 2048;
    static constexpr int CS_OFF = ST_OFF + 2 * ST_BYTES;  // [128] column-sum exchange
    static constexpr int BAR_OFF = CS_OFF + 512;
    // dP_I staging: one fp32 box of 64 rows x 32 columns (128-byte swizzle)
    static constexpr int DPI_OFF = (BAR_OFF + 256 + 1023) / 1024 * 1024;
    // gate: per-warp row-sum partials [2 pairs][2 warpgroups][4 warps][64 queries]
    static constexpr int RS_OFF = DPI_OFF + 8192;
    static constexpr int SMEM = RS_OFF + 4096 + 1024;
    // TMEM columns: no two accumulators share columns; P^T (packed bf16) sits in
    // the S^T columns, query block q (16 queries) at column 64 (q / 4) + 8 (q % 4)
    static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_AB = 320, T_DQ = 384, T_DPI = 448;
};
static_assert(BCfg::SMEM <= 232448, "shared memory per CTA");

__device__ __forceinline__ void named_barrier(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <bool FOX, typename TO>
__global__ void __launch_bounds__(NT, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                  const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mDO,
                  const __grid_constant__ CUtensorMap mP, const __grid_constant__ CUtensorMap mDQ,
                  const __grid_constant__ CUtensorMap mDPI, BwdTcArgs a)
{
    using C = BCfg;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    uint8_t *sAb = sm + C::AB_OFF, *sV = sm + C::V_OFF, *sDs = sm + C::DS_OFF;
    float *sCs = reinterpret_cast<float *>(sm + C::CS_OFF);
    uint8_t *sDpi = sm + C::DPI_OFF;
    float *sRs = reinterpret_cast<float *>(sm + C::RS_OFF);
    auto stage = [&](int s) { return sm + C::ST_OFF + s * C::ST_BYTES; };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BAR_OFF);
    uint64_t *v_full = bars, *ld_full = bars + 1, *ld_empty = bars + 3, *s_full = bars + 5,
             *p_full = bars + 7, *m2_full = bars + 8, *e_done = bars + 9, *ds_free = bars + 10,
             *mma_done = bars + 12;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 13);

    // key tiles along x: the CTAs of one head run together and share its Q, dO
    // tiles in L2 (heads along x, longest tiles first, measured slower)
    const int J = blockIdx.x, h = blockIdx.y;
    const int nblk = a.nblk, last = nblk - 1, Lp = nblk * BT;
    const int niter = last - J + 1;  // off-diagonal tiles last..J+1, then the diagonal
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, tid = threadIdx.x;
    auto tile_of = [&](int it) { return it == niter - 1 ? J : last - it; };

    if (tid == 0) {
        mbar_init(v_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ld_full[s], 1);
            mbar_init(&ld_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, NEW);
        mbar_init(m2_full, 1);
        mbar_init(e_done, NDR);
        mbar_init(&ds_free[0], 1);
        mbar_init(&ds_free[1], 1);
        mbar_init(mma_done, 1);
        mbar_fence_init();
    }
    if (warp == W_MMA) tmem_alloc(tmem_slot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_expect_tx(v_full, C::TILE);
            tma_load_3d(sV, &mV, 0, J * BT, h, v_full);
            int issued = 0;
            for (int it = 0; it < niter; ++it) {
                const int s = it & 1;
                if (it >= 2 && !mbar_wait(&ld_empty[s], ((it >> 1) - 1) & 1, WAIT_LIMIT_NS)) {
                    if (a.err) atomicCAS(a.err, 0, 11);
                    break;
                }
                const int I = tile_of(it);
                const bool diag = it == niter - 1;
                const bool hasP = !diag && I < last;
                uint8_t *st = stage(s);
                const uint32_t bytes = C::TILE * (diag ? 1 : 3) + (hasP ? 8192 : 0) + 1024;
                mbar_expect_tx(&ld_full[s], bytes);
                if (!diag) {
                    const int row = (int)((h * a.npairs + (long long)I * (I - 1) / 2 + J) * BT);
                    tma_load_2d(st + C::S_KH, &mK, 0, row, &ld_full[s]);
                    tma_load_2d(st + C::S_Q, &mQ, 0, h * Lp + I * BT, &ld_full[s]);
                }
                tma_load_3d(st + C::S_DO, &mDO, 0, I * BT, h, &ld_full[s]);
                if (hasP) tma_load_2d(st + C::S_P, &mP, 0, (h * nblk + I) * D, &ld_full[s]);
                float *rows = reinterpret_cast<float *>(st + C::S_ROW);
                bulk_load(rows, a.lse_p + (long long)h * Lp + I * BT, 512, &ld_full[s]);
                bulk_load(rows + 128, a.delta + (long long)h * Lp + I * BT, 512, &ld_full[s]);
                issued = it + 1;
            }
            for (int it = issued - 2 > 0 ? issued - 2 : 0; it < issued; ++it)
                mbar_wait(&ld_full[it & 1], (it >> 1) & 1, WAIT_LIMIT_NS);
        }
    } else if (warp == W_MMA) {
        // the whole warp runs the issue loop (uniform descriptors); lane 0 issues
        const uint32_t lead = lane == 0;
        {
            const uint32_t idS = idesc_f16(128, 128, AB_F16, 0, 0);
            const uint32_t idDP = idesc_f16(128, 128, AB_BF16, 0, 0);
            const uint32_t idDV = idesc_f16(128, D, AB_BF16, 0, 1);
            const uint32_t idAbP = idesc_f16(128, D, AB_F16, 0, 1);
            const uint32_t idMN = idesc_f16(128, D, AB_F16, 1, 1);
            const uint32_t ab0 = smem_u32(sAb), v0 = smem_u32(sV);
            // MMA 1 of pair it: S^T = Khat Qtil^T (not on the diagonal), dP^T = V dO^T
            auto mma1 = [&](int it) -> bool {
                const int s = it & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&ld_full[s], (it >> 1) & 1, WAIT_LIMIT_NS)))
                    return false;
                fence_after_sync();
                const uint32_t kh0 = smem_u32(stage(s) + C::S_KH), q0 = smem_u32(stage(s) + C::S_Q),
                               do0 = smem_u32(stage(s) + C::S_DO);
                if (it != niter - 1) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss_if(lead, tbase + C::T_S, desc_sw128(kh0 + kk * 32, 16, 1024),
                                  desc_sw128(q0 + kk * 32, 16, 1024), idS, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss_if(lead, tbase + C::T_DP, desc_sw128(v0 + kk * 32, 16, 1024),
                              desc_sw128(do0 + kk * 32, 16, 1024), idDP, kk > 0);
                commit_if(lead, s_full);
                return true;
            };
            bool ok = __all_sync(0xffffffffu, mbar_wait(v_full, 0, WAIT_LIMIT_NS)) && mma1(0);
            for (int it = 0; ok && it < niter; ++it) {
                const int s = it & 1, I = tile_of(it);
                const bool diag = it == niter - 1;
                // this pair's P^T (tensor memory) and dS^T (shared memory) are written
                if (!__all_sync(0xffffffffu, mbar_wait(p_full, it & 1, WAIT_LIMIT_NS))) {
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t kh0 = smem_u32(stage(s) + C::S_KH), q0 = smem_u32(stage(s) + C::S_Q),
                               do0 = smem_u32(stage(s) + C::S_DO), p0 = smem_u32(stage(s) + C::S_P),
                               ds0 = smem_u32(sDs + s * C::DS_BYTES);
                // dV += P^T dO   (K = 128 queries, A from tensor memory)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts_if(lead, tbase + C::T_DV, tbase + C::T_S + 64 * (kk >> 2) + 8 * (kk & 3),
                              desc_sw128(do0 + kk * 2048, 16384, 1024), idDV, (it > 0 || kk > 0));
                // the next pair's MMA 1 overwrites the P^T just read (in issue order)
                if (it + 1 < niter && !mma1(it + 1)) {
                    ok = false;
                    break;
                }
                if (!diag) {
                    // the drain has taken the previous pair's Abar, dQtil, dP_I out
                    if (!__all_sync(0xffffffffu, it == 0 || mbar_wait(e_done, (it - 1) & 1, WAIT_LIMIT_NS))) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    if (I < last) {
                        // dP_I (+)= [Abar | Khat]^T Khat  (rows 0..63 = Abar^T Khat)
                        const uint32_t lbo = kh0 - ab0;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss_if(lead, tbase + C::T_DPI, desc_sw128(ab0 + kk * 2048, lbo, 1024),
                                   desc_sw128(kh0 + kk * 2048, 16384, 1024), idMN, kk > 0);
                        // Abar = Abar_{I+1} P_I
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_ss_if(lead, tbase + C::T_AB, desc_sw128(ab0 + kk * 32, 16, 1024),
                                   desc_sw128(p0 + kk * 2048, 16384, 1024), idAbP, kk > 0);
                    }
                    // Abar += dS^T Qtil   (K = 128 queries)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss_if(lead, tbase + C::T_AB, desc_sw128(ds0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                               desc_sw128(q0 + kk * 2048, 16384, 1024), idAbP, (I < last || kk > 0));
                    // dQtil = dS Khat   (A = dS^T read MN-major, K = 128 keys)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss_if(lead, tbase + C::T_DQ, desc_sw128(ds0 + kk * 2048, 16384, 1024),
                               desc_sw128(kh0 + kk * 2048, 16384, 1024), idMN, kk > 0);
                }
                commit_if(lead, m2_full);
                commit_if(lead, &ld_empty[s]);  // the stage's operands are read once these complete
            }
            if (!ok && lead && a.err) atomicCAS(a.err, 0, 12);
            // every MMA this warp issued completes before the CTA frees tensor memory
            commit_if(lead, mma_done);
            if (!__all_sync(0xffffffffu, mbar_wait(mma_done, 0, WAIT_LIMIT_NS)) && lead && a.err)
                atomicCAS(a.err, 0, 15);
        }
    } else if (warp < W_DRAIN0) {
        // softmax warpgroups: warpgroup g takes query columns [64g, 64g + 64);
        // thread j owns key row j of tile J. Per query i the rows hold
        // nb_i = (c_i - lse_i) log2(e) and scale * delta_i.
        const int g = warp >> 2, j = tid & 127;
        const int gj = J * BT + j;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float k1 = a.scale * LOG2E;
        const float cj2 = FOX ? a.c[(long long)h * Lp + gj] * LOG2E : 0.f;
        float colsum = 0.f;
        bool ok = true, ds_late = false;
        for (int it = 0; it < niter; ++it) {
            const int s = it & 1, I = tile_of(it);
            const bool diag = it == niter - 1;
            // s_full: this pair's S^T / dP^T are in tensor memory, and the previous pair's
            // dV products, which read P^T from the columns written below, have completed
            if (ok && (!mbar_wait(&ld_full[s], (it >> 1) & 1, WAIT_LIMIT_NS) ||
                       !mbar_wait(s_full, it & 1, WAIT_LIMIT_NS)))
                ok = false;
            ok = __all_sync(0xffffffffu, ok);  // shuffles and TMEM accesses below are warp-wide
            fence_after_sync();
            const float *rows = reinterpret_cast<const float *>(stage(s) + C::S_ROW);
            const float *sd = a.Sd + ((long long)h * nblk + J) * BT * BT;
            float *dsd = a.dSd + ((long long)h * nblk + J) * BT * BT;
            uint8_t *sDsb = sDs + s * C::DS_BYTES;
            // one 16-column chunk: sv / dp hold S and dP on entry, P and dS on exit
            auto chunk = [&](auto dg, int c, float (&sv)[16], float (&dp)[16]) {
                constexpr bool DG = decltype(dg)::value;
                const float4 *nb4 = reinterpret_cast<const float4 *>(rows + c);
                const float4 *sd4 = reinterpret_cast<const float4 *>(rows + 128 + c);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 nb = nb4[q], sdl = sd4[q];
                    const float nbv[4] = {nb.x, nb.y, nb.z, nb.w}, sdv[4] = {sdl.x, sdl.y, sdl.z, sdl.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int u = 4 * q + e, i = c + u;
                        const float x = fmaf(sv[u], k1, FOX ? nbv[e] - cj2 : nbv[e]);
                        float p = ex2(x);
                        if (DG && i < j) p = 0.f;
                        const float ds = p * fmaf(dp[u], a.scale, -sdv[e]);
                        sv[u] = p;
                        dp[u] = ds;
                        if (DG) dsd[(long long)i * BT + j] = ds;
                    }
                }
                uint32_t pb[8], db[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const __nv_bfloat162 bb = __floats2bfloat162_rn(sv[2 * k], sv[2 * k + 1]);
                    pb[k] = *reinterpret_cast<const uint32_t *>(&bb);
                    const __half2 hh = __floats2half2_rn(dp[2 * k], dp[2 * k + 1]);
                    db[k] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                // P^T of these 16 queries: 8 packed columns, inside the S^T columns this
                // warpgroup has already read
                tmem_st8(tbase + C::T_S + 64 * g + ((c & 63) >> 1) + lane_off, pb);
                // before the first dS^T store: the drain's staging of pair it - 2 has
                // left this buffer (a wait that gives up flags the error; the stores go on)
                if ((c & 63) == 0 && it >= 2 && !mbar_wait(&ds_free[s], ((it >> 1) - 1) & 1, WAIT_LIMIT_NS))
                    ds_late = true;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t off = (c >> 6) * 16384 + sw128_offset(j, (c & 63) + 8 * hf);
                    *reinterpret_cast<uint4 *>(sDsb + off) =
                        make_uint4(db[4 * hf], db[4 * hf + 1], db[4 * hf + 2], db[4 * hf + 3]);
                }
                if (FOX) {
                    // gate: row and column sums of the same fp16-rounded dS that the
                    // MMAs read, so the crossing sums in the gate gradient cancel
                    float *dsv = dp;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float2 f2 = __half22float2(*reinterpret_cast<const __half2 *>(&db[k]));
                        dsv[2 * k] = f2.x;
                        dsv[2 * k + 1] = f2.y;
                        colsum += f2.x + f2.y;
                    }
                    // reduce-scatter over the warp's 32 keys: lanes 2m, 2m+1 end with query c + m
#pragma unroll
                    for (int o = 16, n = 16; o >= 2; o >>= 1, n >>= 1) {
                        const bool up = lane & o;
#pragma unroll
                        for (int k = 0; k < n / 2; ++k) {
                            const float send = up ? dsv[k] : dsv[k + n / 2];
                            const float keep = up ? dsv[k + n / 2] : dsv[k];
                            dsv[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    }
                    dsv[0] += __shfl_xor_sync(0xffffffffu, dsv[0], 1);
                    // this warp's 32 keys' part of query c + m's row sum, combined with
                    // the other three warps' after the pass
                    if (!(lane & 1)) sRs[(((it & 1) * 2 + g) * 4 + (warp & 3)) * 64 + (c & 63) + (lane >> 1)] = dsv[0];
                }
            };
            // the four chunks of this warpgroup, the next chunk's loads in flight while
            // one is computed; the diagonal tile (logits from the UT prep, causal mask,
            // dS also to the prep's adjoint) is its own instantiation
            auto pass = [&](auto dg) {
                constexpr bool DG = decltype(dg)::value;
                float sv[2][16], dp[2][16];
                auto load = [&](int b, int c) {
                    if (DG) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) sv[b][u] = sd[(c + u) * BT + j];
                    } else {
                        tmem_ld16(tbase + C::T_S + c + lane_off, sv[b]);
                    }
                    tmem_ld16(tbase + C::T_DP + c + lane_off, dp[b]);
                };
                load(0, 64 * g);
                tmem_wait_ld_tied(sv[0], dp[0]);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int b = q4 & 1, c = 64 * g + 16 * q4;
                    if (q4 < 3) load(b ^ 1, c + 16);
                    chunk(dg, c, sv[b], dp[b]);
                    if (q4 < 3) tmem_wait_ld_tied(sv[b ^ 1], dp[b ^ 1]);
                }
            };
            if (ok) {
                if (diag)
                    pass(std::true_type{});
                else
                    pass(std::false_type{});
            }
            if (FOX) {
                // the row sums of dS over the tile's 128 keys: one atomic per query
                named_barrier(4 + g, 128);
                if (ok && j < 64) {
                    const float *rs = sRs + ((it & 1) * 2 + g) * 4 * 64 + j;
                    atomicAdd(a.rowsum + (long long)h * Lp + I * BT + 64 * g + j,
                              (rs[0] + rs[64] + rs[128] + rs[192]) / a.scale);
                }
            }
            tmem_wait_st();
            fence_async_smem();
            fence_before_sync();
            mbar_arrive(p_full);
        }
        // column sums: warpgroup 1 hands its half to warpgroup 0
        if (g == 1) sCs[j] = colsum;
        named_barrier(1, NEW);
        if ((!ok || ds_late) && a.err) atomicCAS(a.err, 0, 13);
        if (ok && g == 0 && a.colsum && gj < a.L) a.colsum[(long long)h * Lp + gj] = (colsum + sCs[j]) / a.scale;
    } else if (warp < W_PROD) {
        // drain warpgroup: thread j = lane j of TMEM (key row for Abar and dV, query
        // row for dQtil, row f < 64 of dP_I); all 64 columns of each result.
        // dQtil leaves through fp32 staging (128B-swizzled boxes of 32 columns) in
        // this pair's dS^T buffer, spent once MMA 2 has completed, and bulk tensor
        // reduce-add; the buffer goes back to the softmax after the reduction has
        // read it. dP_I leaves the same way through its own 8 KB staging box.
        const int j = tid - 32 * W_DRAIN0;
        const int gj = J * BT + j;
        const bool leader = j == 0;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float dpv[2][32];  // this thread's row of dP_I
        bool ok = true;
        for (int it = 0; it < niter; ++it) {
            const int s = it & 1, I = tile_of(it);
            const bool diag = it == niter - 1;
            if (ok && !mbar_wait(m2_full, it & 1, WAIT_LIMIT_NS)) ok = false;
            ok = __all_sync(0xffffffffu, ok);  // TMEM loads below are warp-wide
            fence_after_sync();
            uint8_t *stq = sDs + s * C::DS_BYTES;  // dQtil: 2 x 16 KB
            const bool drain = ok && !diag;
            if (drain) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    // dQtil rows of tile I (lane = query row)
                    float v[32];
                    tmem_ld32(tbase + C::T_DQ + c0 + lane_off, v);
                    uint8_t *box = stq + (c0 >> 5) * 16384 + j * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        *reinterpret_cast<float4 *>(box + ((k ^ (j & 7)) << 4)) =
                            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                }
                fence_async_smem();
            }
            named_barrier(2, NDR);  // every staging row written: the reduction starts first
            if (leader && drain) {
                tma_reduce_add_2d(&mDQ, 0, h * Lp + I * BT, stq);
                tma_reduce_add_2d(&mDQ, 32, h * Lp + I * BT, stq + 16384);
                bulk_commit();
            }
            if (drain) {
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    // chain adjoint: operand for the next pair, or dKtil_J after pair (J+1, J)
                    float v[32];
                    tmem_ld32(tbase + C::T_AB + c0 + lane_off, v);
                    if (I > J + 1) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 u;
                            __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                            for (int k = 0; k < 4; ++k) hh[k] = __floats2half2_rn(v[q * 8 + 2 * k], v[q * 8 + 2 * k + 1]);
                            *reinterpret_cast<uint4 *>(sAb + sw128_offset(j, c0 + q * 8)) = u;
                        }
                    } else {
                        float *dk = a.dKt + ((long long)h * Lp + gj) * D + c0;
#pragma unroll
                        for (int u = 0; u < 32; u += 4)
                            *reinterpret_cast<float4 *>(dk + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
                    }
                }
                if (I < last) {
                    // dP_I rows f = 0..63 live in lanes 0..63 (the first two warps);
                    // they leave by atomics once the tensor memory is released
                    tmem_ld32(tbase + C::T_DPI + lane_off, dpv[0]);
                    tmem_ld32(tbase + C::T_DPI + 32 + lane_off, dpv[1]);
                }
                fence_async_smem();
            }
            // TMEM results read and Abar written: MMA 2 of the next pair may go
            fence_before_sync();
            mbar_arrive(e_done);
            if (I < last && j < D) {
                // dP_I (rows j < 64: the first two drain warps) leaves by bulk tensor
                // reduce-add, 32 columns at a time through one 8 KB staging box
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    if (drain) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4 *>(sDpi + j * 128 + ((k ^ (j & 7)) << 4)) =
                                make_float4(dpv[hb][4 * k], dpv[hb][4 * k + 1], dpv[hb][4 * k + 2], dpv[hb][4 * k + 3]);
                        fence_async_smem();
                    }
                    named_barrier(3, 64);  // the box is written
                    if (leader && drain) {
                        tma_reduce_add_2d(&mDPI, 32 * hb, (h * nblk + I) * D, sDpi);
                        bulk_commit();
                        bulk_wait_read<0>();
                    }
                    named_barrier(3, 64);  // and read: it may be written again
                }
            }
            if (leader) {
                if (drain) bulk_wait_read<0>();
                mbar_arrive(&ds_free[s]);  // the softmax may write this dS^T buffer again
            }
        }
        if (leader) bulk_wait_all();
        // the last tile has no off-diagonal pairs: its dKtil is zero
        if (ok && J == last) {
            float *dk = a.dKt + ((long long)h * Lp + gj) * D;
            for (int e = 0; e < D; e += 4) *reinterpret_cast<float4 *>(dk + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // dV_J, complete after the last MMA 2 (waited for above)
        if (ok) {
            TO *dst = static_cast<TO *>(a.dv) + ((long long)h * a.L + gj) * D;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                float v[32];
                tmem_ld32(tbase + C::T_DV + c0 + lane_off, v);  // warp-wide; rows past L drop
                if (gj < a.L) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) dst[c0 + e] = from_f<TO>(v[e]);
                }
            }
        } else if (a.err) {
            atomicCAS(a.err, 0, 14);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == W_MMA) tmem_dealloc(tbase, 512);
}

// Per-query terms of the tensor-core backward: nb = (c - lse) log2(e) (+inf
// lse past L gives nb = -inf, probability 0) and delta scaled in place.
__global__ void row_terms_kernel(const float *lse, const float *c, float *nb, float *delta,
                                 float scale, int L, int Lp, int nh)
{
    const long long n = (long long)nh * Lp;
    for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < n;
         x += (long long)gridDim.x * blockDim.x) {
        const int h = (int)(x / Lp), i = (int)(x % Lp);
        nb[x] = i < L ? ((c ? c[x] : 0.f) - lse[(long long)h * L + i]) * LOG2E : -INFINITY;
        delta[x] *= scale;
    }
}

// bf16 copy of an fp32 tensor (the dO operand when out/dout are fp32)
__global__ void f32_to_bf16_kernel(const float *src, bf16 *dst, long long n)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

template <bool FOX, typename TO>
cudaError_t launch(const CUtensorMap *m, const BwdTcArgs &a, cudaStream_t st)
{
    auto k = bwd_tc_kernel<FOX, TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg::SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nblk, a.nh), NT, BCfg::SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], a);
    count_launches();
    return cudaGetLastError();
}

}  // namespace

bool attn_bwd_tc_supported(Types t, int d) { return t.in == BF16 && t.mid == F16 && d == 64; }

cudaError_t attn_bwd_tc_prepare(const BwdArgs &b, Types t, int d, float *lse_p, void *dout_bf16,
                                cudaStream_t st)
{
    const int Lp = b.nblk * BT;
    // delta is scratch of the backward: scaled here in place for the kernel
    row_terms_kernel<<<592, 256, 0, st>>>(b.lse, b.c, lse_p, b.delta, b.scale, b.L, Lp, b.nh);
    count_launches();
    if (t.out == F32) {
        const long long n = (long long)b.nh * b.L * d;
        f32_to_bf16_kernel<<<1184, 256, 0, st>>>(static_cast<const float *>(b.dout),
                                                 static_cast<bf16 *>(dout_bf16), n);
        count_launches();
    }
    return cudaGetLastError();
}

cudaError_t attn_bwd_tc(const BwdArgs &b, Types t, float *lse_p, void *dout_bf16, int *err,
                        cudaStream_t st)
{
    const int Lp = b.nblk * BT;
    const long long npairs = (long long)b.nblk * (b.nblk - 1) / 2;
    const void *dob = t.out == F32 ? dout_bf16 : b.dout;
    CUtensorMap m[7];
    if (!make_map_2d(&m[0], b.Qt, F16, D, (uint64_t)b.nh * Lp, 128)) return cudaErrorInvalidValue;
    if (npairs > 0) {
        if (!make_map_2d(&m[1], b.Khat, F16, D, (uint64_t)b.nh * npairs * BT, 128)) return cudaErrorInvalidValue;
    } else {
        m[1] = m[0];
    }
    if (!make_map_3d(&m[2], b.v, BF16, D, b.L, b.nh, 128) ||
        !make_map_3d(&m[3], dob, BF16, D, b.L, b.nh, 128) ||
        !make_map_2d(&m[4], b.Pm, F16, D, (uint64_t)b.nh * b.nblk * D, D) ||
        !make_map_f32_2d(&m[5], b.dQt, D, (uint64_t)b.nh * Lp, 128) ||
        !make_map_f32_2d(&m[6], b.dPm, D, (uint64_t)b.nh * b.nblk * D, D))
        return cudaErrorInvalidValue;
    BwdTcArgs a{b.Sd, b.c, lse_p, b.delta, b.scale, b.L, b.nblk, b.nh, npairs,
                b.dQt, b.dKt, b.dPm, b.dSd, b.dv, b.rowsum, b.colsum, err};
    const bool fox = b.c != nullptr;
    if (t.out == F32) return fox ? launch<true, float>(m, a, st) : launch<false, float>(m, a, st);
    return fox ? launch<true, bf16>(m, a, st) : launch<false, bf16>(m, a, st);
}

}  // namespace path
