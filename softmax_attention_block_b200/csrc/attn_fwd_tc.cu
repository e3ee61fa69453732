// PaTH attention forward on 5th-generation tensor cores (sm_100a).
//
// One CTA per (128-row query tile I, head). Warp roles:
//   warps 0-7  softmax: warps w and w+4 share TMEM lanes 32(w%4)..+31 (query
//              rows); each takes half of the 128 key columns of S and half of
//              the d columns of O, exchanging the row max through shared
//              memory, so each SM sub-partition interleaves two softmax warps
//   warp 8     producer: TMA loads of Qtil_I, then per key tile the transported
//              keys Khat_{I,J}, the values V_J and the gate prefix c_J into a
//              ring of NS stages
//   warp 9     MMA issuer: S = Qtil Khat^T and O_tile = P V (fp16 operands,
//              fp32 accumulators in TMEM; S double-buffered). P lies in [0, 1],
//              where fp16 keeps three more mantissa bits than bf16, so V is
//              read from an fp16 copy made once per call.
// The diagonal tile's logits come precomputed from the UT prep (the
// full-matrix form of each block); tiles J < I come from S = Qtil Khat^T.
// Softmax works in the log2 domain; the running max rescales the register
// accumulator when each P.V tile is added. At head dim 64 P and the P.V tiles
// are double-buffered: a tile's P.V is added two tiles later and S runs two
// tiles ahead, so the softmax never waits for the P.V just issued.
#include "attn.cuh"
#include "attn_tc.cuh"
#include "runtime.cuh"
#include "tc.cuh"

namespace path {

namespace {

using namespace tc;

constexpr int NT = 320;
constexpr int W_PROD = 8, W_MMA = 9;
constexpr int NSOFT = 256;  // softmax threads
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

template <int D>
struct Cfg {
    static constexpr int PANELS = D / 64;
    static constexpr int TILE = 128 * D * 2;  // bytes of one 128-row 16-bit tile
    static constexpr int NS = D == 64 ? 3 : 2;
    // P buffers in shared memory and P.V tiles in TMEM: with two, a tile's P.V is
    // folded into the accumulator two tiles later and S runs two tiles ahead
    static constexpr int PB = D == 64 ? 2 : 1;
    static constexpr int Q_OFF = 0;
    static constexpr int ST_OFF = Q_OFF + TILE;
    static constexpr int ST_BYTES = 2 * TILE + 1024;  // K, V, gate prefix (512 B)
    static constexpr int P_OFF = ST_OFF + NS * ST_BYTES;
    static constexpr int BAR_OFF = P_OFF + PB * 128 * 128 * 2;
    static constexpr int RED_OFF = BAR_OFF + 256;     // [2][2][128] row maxima, [2][128] row sums
    static constexpr int SMEM = RED_OFF + 6 * 128 * 4 + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128) S1 [128,256) O_b [256 + b D, 256 + (b+1) D)
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void named_barrier(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ void flag_error(int *err, int code)
{
    if (err) atomicCAS(err, 0, code);
}

template <typename TO>
__device__ __forceinline__ void store_row(TO *dst, const float *v, int D, float scale);

template <>
__device__ __forceinline__ void store_row<float>(float *dst, const float *v, int D, float scale)
{
    for (int e = 0; e < D; e += 4)
        *reinterpret_cast<float4 *>(dst + e) =
            make_float4(v[e] * scale, v[e + 1] * scale, v[e + 2] * scale, v[e + 3] * scale);
}

template <>
__device__ __forceinline__ void store_row<bf16>(bf16 *dst, const float *v, int D, float scale)
{
    for (int e = 0; e < D; e += 8) {
        uint4 u;
        __nv_bfloat162 *hh = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) hh[i] = __floats2bfloat162_rn(v[e + 2 * i] * scale, v[e + 2 * i + 1] * scale);
        *reinterpret_cast<uint4 *>(dst + e) = u;
    }
}

template <int D, bool FOX, typename TO>
__global__ void __launch_bounds__(NT, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                  const __grid_constant__ CUtensorMap mV, FwdTcArgs a)
{
    using C = Cfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BAR_OFF);
    uint64_t *q_full = bars;
    uint64_t *kv_full = bars + 1;
    uint64_t *kv_empty = bars + 1 + NS;
    uint64_t *s_full = bars + 1 + 2 * NS;
    // P of tile it is complete when p_full[it & 1] completes. One barrier per
    // parity: a warp pair may finish tile it + 1 (its S and the P.V it folds are
    // ready) before another pair has finished tile it, and its arrival must not
    // count toward tile it's phase.
    uint64_t *p_full = bars + 3 + 2 * NS;  // [2]
    uint64_t *o_full = bars + 5 + 2 * NS;  // [PB]
    uint64_t *mma_done = bars + 5 + 2 * NS + C::PB;  // every MMA of the CTA completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6 + 2 * NS + C::PB);
    uint8_t *sQ = sm + C::Q_OFF;
    uint8_t *sP = sm + C::P_OFF;
    auto sK = [&](int s) { return sm + C::ST_OFF + s * C::ST_BYTES; };
    auto sV = [&](int s) { return sm + C::ST_OFF + s * C::ST_BYTES + C::TILE; };
    auto sC = [&](int s) { return reinterpret_cast<float *>(sm + C::ST_OFF + s * C::ST_BYTES + 2 * C::TILE); };

    // heads along x: blocks start in launch order, so every head's longest rows of
    // the causal triangle start first
    const int I = a.nblk - 1 - (int)blockIdx.y;
    const int h = blockIdx.x;
    const int niter = I + 1;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int Lp = a.nblk * BT;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&p_full[0], NSOFT);
        mbar_init(&p_full[1], NSOFT);
        for (int b = 0; b < C::PB; ++b) mbar_init(&o_full[b], 1);
        mbar_init(mma_done, 1);
        mbar_fence_init();
    }
    if (warp == W_MMA) tmem_alloc(tmem_slot, C::TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == W_PROD) {
        if (lane == 0) {
            int issued = 0, withheld = -1;
            mbar_expect_tx(q_full, C::TILE);
            for (int p = 0; p < C::PANELS; ++p)
                tma_load_2d(sQ + p * 16384, &mQ, 64 * p, h * Lp + I * BT, q_full);
            for (int it = 0; it < niter; ++it) {
                const int s = it % NS;
                if (it >= NS && !mbar_wait(&kv_empty[s], ((it / NS) - 1) & 1, a.limit_ns)) {
                    flag_error(a.err, 1);
                    break;
                }
                if (a.withhold && I == a.nblk - 1 && it == 1) {
                    withheld = it;  // test hook: this stage's copies are never issued
                    continue;
                }
                const int J = it == 0 ? I : I - it;
                const uint32_t bytes = C::TILE + (it > 0 ? C::TILE : 0) + (FOX ? 512 : 0);
                mbar_expect_tx(&kv_full[s], bytes);
                if (it > 0) {
                    const int row = (int)((h * a.npairs + (long long)I * (I - 1) / 2 + J) * BT);
                    for (int p = 0; p < C::PANELS; ++p)
                        tma_load_2d(sK(s) + p * 16384, &mK, 64 * p, row, &kv_full[s]);
                }
                for (int p = 0; p < C::PANELS; ++p)
                    tma_load_3d(sV(s) + p * 16384, &mV, 64 * p, J * BT, h, &kv_full[s]);
                if (FOX) bulk_load(sC(s), a.c + (long long)h * Lp + J * BT, 512, &kv_full[s]);
                issued = it + 1;
            }
            // never leave while copies into this CTA's shared memory are in flight:
            // wait for every stage whose copies were issued (the copies complete on
            // their own; the bound is the rule for every wait, set far above them)
            for (int it = issued - NS > 0 ? issued - NS : 0; it < issued; ++it)
                if (it != withheld) mbar_wait(&kv_full[it % NS], (it / NS) & 1, 8 * a.limit_ns);
        }
    } else if (warp == W_MMA) {
        if (lane == 0) {
            const uint32_t idS = idesc_f16(128, 128, AB_F16, 0, 0);
            const uint32_t idO = idesc_f16(128, D, AB_F16, 0, 1);
            const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            bool ok = mbar_wait(q_full, 0, a.limit_ns) && mbar_wait(&kv_full[0], 0, a.limit_ns);
            fence_after_sync();
            // S = Qtil Khat^T of tile n into S buffer n & 1 (tile 0, the diagonal,
            // takes its logits from the UT prep)
            auto issue_s = [&](int n) -> bool {
                const int s = n % NS, b = n & 1;
                if (!mbar_wait(&kv_full[s], (n / NS) & 1, a.limit_ns)) return false;
                fence_after_sync();
                const uint32_t k_addr = smem_u32(sK(s));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
                    mma_ss(tbase + b * 128, desc_sw128(q_addr + off, 16, 1024),
                           desc_sw128(k_addr + off, 16, 1024), idS, kk > 0);
                }
                commit(&s_full[b]);
                return true;
            };
            // O_tile(it) = P(it) V(it) into P.V buffer it % PB
            auto issue_pv = [&](int it) {
                const int s = it % NS, pb = it % C::PB;
                const uint32_t v_addr = smem_u32(sV(s)), pa = p_addr + pb * 32768;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk / 4) * 16384 + (kk % 4) * 32;
                    mma_ss(tbase + 256 + pb * D, desc_sw128(pa + aoff, 16, 1024),
                           desc_sw128(v_addr + kk * 2048, 16384, 1024), idO, kk > 0);
                }
                commit(&o_full[pb]);
                commit(&kv_empty[s]);
            };
            if (NS >= 3) {
                // S two tiles ahead: S(it + 2) reuses the S buffer of tile it right
                // after tile it's softmax, and its keys were loaded a tile earlier
                for (int n = 1; ok && n <= 2 && n < niter; ++n) ok = issue_s(n);
                for (int it = 0; ok && it < niter; ++it) {
                    if (!mbar_wait(&p_full[it & 1], (it >> 1) & 1, a.limit_ns)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    issue_pv(it);
                    if (it >= 1 && it + 2 < niter && !issue_s(it + 2)) ok = false;
                }
            } else {
                // S one tile ahead, overlapping this tile's softmax
                for (int it = 0; ok && it < niter; ++it) {
                    if (it + 1 < niter && !issue_s(it + 1)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(&p_full[it & 1], (it >> 1) & 1, a.limit_ns)) {
                        ok = false;
                        break;
                    }
                    fence_after_sync();
                    issue_pv(it);
                }
            }
            if (!ok) flag_error(a.err, 2);
            // the tensor memory is freed after this warp leaves: no MMA it issued
            // may still be running then (on the normal path they all completed)
            commit(mma_done);
            mbar_wait(mma_done, 0, 8 * a.limit_ns);
        }
    } else {
        // softmax: row r = TMEM lane; this warp owns S columns [c0s, c0s+64) and
        // O columns [c0o, c0o+D/2) of it
        constexpr int DH = D / 2;
        const int q4 = warp & 3, hf = warp >> 2;
        const int r = q4 * 32 + lane;
        const int gi = I * BT + r;
        const bool valid = gi < a.L;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const int c0s = hf * 64, c0o = hf * DH;
        float *red = reinterpret_cast<float *>(sm + C::RED_OFF);  // [2][2][128]
        float *redl = red + 512;                                  // [2][128]
        const float k1 = a.scale_log2;
        const float ci2 = FOX ? a.c[(long long)h * Lp + gi] * LOG2E : 0.f;
        // without the gate and with a positive scale, the logits stay unscaled: the
        // row max scales after the fact and the scale joins the exponent's FFMA
        const bool fast = !FOX && k1 > 0.f;
        const float kx = fast ? k1 : 1.f;
        float acc[DH];
#pragma unroll
        for (int e = 0; e < DH; ++e) acc[e] = 0.f;
        float m = -INFINITY, l = 0.f, mA = -INFINITY;
        float mh0 = -INFINITY, mh1 = -INFINITY;  // row max of the tiles in P.V buffers 0, 1
        bool ok = true;
        const float *sd = a.Sd + (((long long)h * a.nblk + I) * BT + r) * BT + c0s;
        // Every thread runs every iteration and every named barrier; after a
        // failed wait the work is skipped, never the barriers.
        for (int it = 0; it < niter; ++it) {
            const int s = it % NS, b = it & 1;
            if (ok && FOX && !mbar_wait(&kv_full[s], (it / NS) & 1, a.limit_ns)) ok = false;
            const float *cj = sC(s) + c0s;
            float z[64];
            float pmax = -INFINITY;
            if (ok && it > 0 && !mbar_wait(&s_full[b], ((it - 1) >> 1) & 1, a.limit_ns)) ok = false;
            ok = __all_sync(0xffffffffu, ok);  // TMEM loads below are warp-wide
            if (ok) {
                if (it == 0) {
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const float4 v4 = *reinterpret_cast<const float4 *>(sd + j);
                        z[j] = v4.x;
                        z[j + 1] = v4.y;
                        z[j + 2] = v4.z;
                        z[j + 3] = v4.w;
                    }
                } else {
                    fence_after_sync();
                    float *z0 = z, *z1 = z + 32;
                    tmem_ld32(tbase + b * 128 + c0s + lane_off, *reinterpret_cast<float(*)[32]>(z0));
                    tmem_ld32(tbase + b * 128 + c0s + 32 + lane_off, *reinterpret_cast<float(*)[32]>(z1));
                }
                if (it == 0) {  // the diagonal tile: causal mask
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const float bias = FOX ? ci2 - cj[j] * LOG2E : 0.f;
                        const float t = fast ? z[j] : fmaf(z[j], k1, bias);
                        z[j] = c0s + j <= r ? t : -INFINITY;
                    }
                } else if (!fast) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const float bias = FOX ? ci2 - cj[j] * LOG2E : 0.f;
                        z[j] = fmaf(z[j], k1, bias);
                    }
                }
#pragma unroll
                for (int j = 0; j < 64; j += 2) pmax = fmax3(pmax, z[j], z[j + 1]);
                if (fast) pmax *= k1;
            }
            float *rb = red + (it & 1) * 256;
            rb[hf * 128 + r] = pmax;
            named_barrier(1 + q4, 64);
            const float m_new = fmaxf(m, fmaxf(rb[r], rb[128 + r]));
            // fold the P.V of tile it - PB (scaled to that tile's max) into the
            // accumulator; its P buffer is then free for this tile's probabilities
            if (it >= C::PB) {
                const int t = it - C::PB, pb = t % C::PB;
                if (ok && !mbar_wait(&o_full[pb], (t / C::PB) & 1, a.limit_ns)) ok = false;
                ok = __all_sync(0xffffffffu, ok);  // TMEM loads below are warp-wide
                if (ok) {
                    fence_after_sync();
                    const float mt = pb == 0 ? mh0 : mh1;
                    const float corr = ex2(mA - mt);
#pragma unroll
                    for (int c0 = 0; c0 < DH; c0 += 32) {
                        float v[32];
                        tmem_ld32(tbase + 256 + pb * D + c0o + c0 + lane_off, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) acc[c0 + j] = fmaf(acc[c0 + j], corr, v[j]);
                    }
                    mA = mt;
                }
            }
            if (ok) {
                // probabilities -> P buffer it % PB (fp16, swizzled K-major panel hf)
                // and partial row sum
                uint8_t *pbuf = sP + (it % C::PB) * 32768 + hf * 16384;
                float rowsum = 0.f;
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint4 u;
                    __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const float p0 = ex2(fmaf(z[g * 8 + 2 * q2], kx, -m_new));
                        const float p1 = ex2(fmaf(z[g * 8 + 2 * q2 + 1], kx, -m_new));
                        rowsum += p0 + p1;
                        hh[q2] = __floats2half2_rn(p0, p1);
                    }
                    *reinterpret_cast<uint4 *>(pbuf + sw128_offset(r, g * 8)) = u;
                }
                l = fmaf(l, ex2(m - m_new), rowsum);
                m = m_new;
                if (it % C::PB == 0)
                    mh0 = m_new;
                else
                    mh1 = m_new;
            }
            fence_async_smem();
            fence_before_sync();
            mbar_arrive(&p_full[it & 1]);
        }
        // the last PB tiles' P.V
        for (int t = niter - C::PB > 0 ? niter - C::PB : 0; t < niter; ++t) {
            const int pb = t % C::PB;
            if (ok && !mbar_wait(&o_full[pb], (t / C::PB) & 1, a.limit_ns)) ok = false;
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                fence_after_sync();
                const float mt = pb == 0 ? mh0 : mh1;
                const float corr = ex2(mA - mt);
#pragma unroll
                for (int c0 = 0; c0 < DH; c0 += 32) {
                    float v[32];
                    tmem_ld32(tbase + 256 + pb * D + c0o + c0 + lane_off, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c0 + j] = fmaf(acc[c0 + j], corr, v[j]);
                }
                mA = mt;
            }
        }
        // row sum: both halves share the running max, so the partial sums add
        redl[hf * 128 + r] = l;
        named_barrier(1 + q4, 64);
        const float lt = redl[r] + redl[128 + r];
        if (!ok) flag_error(a.err, 3);
        if (valid) {
            TO *dst = static_cast<TO *>(a.out) + ((long long)h * a.L + gi) * D + c0o;
            const float inv = ok ? 1.f / lt : __int_as_float(0x7fc00000);
            store_row<TO>(dst, acc, DH, inv);
            if (hf == 0) a.lse[(long long)h * a.L + gi] = ok ? (m + log2f(lt)) * LN2 : __int_as_float(0x7fc00000);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == W_MMA) tmem_dealloc(tbase, C::TMEM_COLS);
}

template <int D, bool FOX, typename TO>
cudaError_t launch(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                   const FwdTcArgs &a, cudaStream_t st)
{
    auto k = fwd_tc_kernel<D, FOX, TO>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<dim3(a.nh, a.nblk), NT, Cfg<D>::SMEM, st>>>(mQ, mK, mV, a);
    count_launches();
    return cudaGetLastError();
}

// dst = fp16 copy of src (bf16), 8 elements per thread step
__global__ void to_f16_kernel(const bf16 *src, f16 *dst, long long n8)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
         i += (long long)gridDim.x * blockDim.x) {
        const uint4 u = reinterpret_cast<const uint4 *>(src)[i];
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
        uint4 o;
        __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
        for (int k = 0; k < 4; ++k) h[k] = __float22half2_rn(__bfloat1622float2(b[k]));
        reinterpret_cast<uint4 *>(dst)[i] = o;
    }
}

}  // namespace

cudaError_t convert_to_f16(const void *src, void *dst, long long n, cudaStream_t st)
{
    if (n % 8) return cudaErrorInvalidValue;
    to_f16_kernel<<<1184, 256, 0, st>>>(static_cast<const bf16 *>(src), static_cast<f16 *>(dst), n / 8);
    count_launches();
    return cudaGetLastError();
}

bool attn_fwd_tc_supported(Types t, int d)
{
    return t.in == BF16 && t.mid == F16 && (d == 64 || d == 128);
}

cudaError_t attn_fwd_tc(const FwdArgs &f, Types t, int d, int *err, cudaStream_t st)
{
    const int Lp = f.nblk * BT;
    const long long npairs = (long long)f.nblk * (f.nblk - 1) / 2;
    CUtensorMap mQ, mK, mV;
    if (!make_map_2d(&mQ, f.Qt, F16, d, (uint64_t)f.nh * Lp, 128)) return cudaErrorInvalidValue;
    if (npairs > 0) {
        if (!make_map_2d(&mK, f.Khat, F16, d, (uint64_t)f.nh * npairs * BT, 128))
            return cudaErrorInvalidValue;
    } else {
        mK = mQ;  // no off-diagonal tiles: never read
    }
    if (!make_map_3d(&mV, f.vh, F16, d, f.L, f.nh, 128)) return cudaErrorInvalidValue;
    const int withhold = withhold_kv_load() && f.nblk > 1;
    FwdTcArgs a{f.Sd, f.c, f.scale * 1.4426950408889634f, f.L, f.nblk, f.nh, npairs, f.out, f.lse, err,
                withhold ? 2000000ull : WAIT_LIMIT_NS, withhold};
    const bool fox = f.c != nullptr;
    const bool f32 = t.out == F32;
#define L_(D_, FOX_, TO_) return launch<D_, FOX_, TO_>(mQ, mK, mV, a, st)
    if (d == 64) {
        if (fox) { if (f32) L_(64, true, float); else L_(64, true, bf16); }
        else { if (f32) L_(64, false, float); else L_(64, false, bf16); }
    } else {
        if (fox) { if (f32) L_(128, true, float); else L_(128, true, bf16); }
        else { if (f32) L_(128, false, float); else L_(128, false, bf16); }
    }
#undef L_
}

}  // namespace path
