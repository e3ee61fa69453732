// PaTH attention main loops, fp32 CUDA-core (SIMT) versions: one thread per
// row. These serve the fp32 path and are the reference GPU implementation
// the tensor-core kernels are checked against.
//
// Blockwise view (tiles of BT = 128 positions, block J = [J*BT, (J+1)*BT)):
//   z_ij = scale * Sd_I[i][j] + c_i - c_j                       (j in tile I, j <= i)
//   z_ij = scale * Qtil_i . Khat_{I,J}[j] + c_i - c_j            (j in tile J < I)
// with Khat_{I,J} = Ktil_J P_{J+1}^T ... P_{I-1}^T: the keys of block J as the
// in-place-updated key cache holds them when block I starts (the right-to-left
// transport of gist.science section 3, run on the key side and stored once).
#include "attn.cuh"
#include "runtime.cuh"

namespace path {

namespace {

constexpr int QR = 64;  // query rows per CTA (half a tile)
constexpr int KS = 64;  // key rows staged per step

__device__ __forceinline__ long long pair_index(int I, int J) { return (long long)I * (I - 1) / 2 + J; }

template <typename T, int D>
__device__ void stage_rows(float *dst, int ldd, const T *src, int rows_valid)
{
    for (int e = threadIdx.x; e < KS * D; e += blockDim.x) {
        const int r = e / D, c = e % D;
        dst[r * ldd + c] = r < rows_valid ? to_f(src[(long long)r * D + c]) : 0.f;
    }
}

// ---------------------------------------------------------------------------
// Transport chain: Khat_{I,J} for every pair J < I.
// grid (nblk - 1, nh), BT threads; thread r carries row r of block J.
// ---------------------------------------------------------------------------
template <typename T, int D>  // T: intermediate (mid) type
__global__ void __launch_bounds__(BT) chain_kernel(const T *Kt, const T *Pm, T *Khat, int nblk)
{
    extern __shared__ float sm[];
    float *sP = sm;                 // [D][D]
    float *sX = sm + D * D;         // [BT][D+1]
    const int J = blockIdx.x, h = blockIdx.y, r = threadIdx.x;
    const int Lp = nblk * BT;
    const long long npairs = (long long)nblk * (nblk - 1) / 2;
    const T *kt = Kt + ((long long)h * Lp + (long long)J * BT + r) * D;
    float *x = sX + r * (D + 1);
    for (int e = 0; e < D; ++e) x[e] = to_f(kt[e]);
    for (int I = J + 1; I < nblk; ++I) {
        T *dst = Khat + ((long long)h * npairs + pair_index(I, J)) * BT * D + (long long)r * D;
        for (int e = 0; e < D; ++e) dst[e] = from_f<T>(x[e]);
        if (I + 1 >= nblk) break;
        __syncthreads();
        const T *p = Pm + ((long long)h * nblk + I) * D * D;
        for (int e = threadIdx.x; e < D * D; e += blockDim.x) sP[e] = to_f(p[e]);
        __syncthreads();
        float nx[D];
#pragma unroll 4
        for (int e = 0; e < D; ++e) {
            float s = 0.f;
            for (int f = 0; f < D; ++f) s = fmaf(x[f], sP[e * D + f], s);
            nx[e] = s;
        }
        for (int e = 0; e < D; ++e) x[e] = nx[e];
    }
}

// ---------------------------------------------------------------------------
// Forward. grid (2*nblk, nh), QR threads; thread i = query row.
// ---------------------------------------------------------------------------
template <typename T, typename TM, typename TO, int D>  // input, mid (intermediate), output types
__global__ void __launch_bounds__(QR) fwd_kernel(FwdArgs a)
{
    extern __shared__ float sm[];
    float *sQ = sm;               // [D][QR]   (transposed, own column)
    float *sK = sQ + D * QR;      // [KS][D]
    float *sV = sK + KS * D;      // [KS][D]
    float *sC = sV + KS * D;      // [KS]
    const int I = blockIdx.x / 2, half = blockIdx.x % 2, h = blockIdx.y;
    const int L = a.L, nblk = a.nblk, Lp = nblk * BT;
    const int li = half * QR + threadIdx.x;  // row within tile I
    const int gi = I * BT + li;
    const bool valid = gi < L;
    const TM *qt = static_cast<const TM *>(a.Qt) + ((long long)h * Lp + gi) * D;
    for (int e = 0; e < D; ++e) sQ[e * QR + threadIdx.x] = to_f(qt[e]);
    const float ci = (a.c && valid) ? a.c[(long long)h * Lp + gi] : 0.f;
    float m = -INFINITY, l = 0.f, o[D];
    for (int e = 0; e < D; ++e) o[e] = 0.f;
    const T *V = static_cast<const T *>(a.v) + (long long)h * L * D;

    auto process = [&](const float *z, int cnt, int k0) {
        float mc = m;
        for (int u = 0; u < cnt; ++u) mc = fmaxf(mc, z[u]);
        if (mc == -INFINITY) return;
        const float corr = __expf(m - mc);
        l *= corr;
        for (int e = 0; e < D; ++e) o[e] *= corr;
        m = mc;
        for (int u = 0; u < cnt; ++u) {
            const float p = __expf(z[u] - m);
            l += p;
            const float *vr = sV + (k0 + u) * D;
            for (int e = 0; e < D; ++e) o[e] = fmaf(p, vr[e], o[e]);
        }
    };

    // diagonal tile: keys of tile I, j <= i
    for (int k0 = 0; k0 < BT; k0 += KS) {
        __syncthreads();
        const int rows = min(KS, L - (I * BT + k0));
        stage_rows<T, D>(sV, D, V + (long long)(I * BT + k0) * D, rows);
        for (int u = threadIdx.x; u < KS; u += blockDim.x)
            sC[u] = a.c ? a.c[(long long)h * Lp + I * BT + k0 + u] : 0.f;
        __syncthreads();
        const float *sd = a.Sd + (((long long)h * nblk + I) * BT + li) * BT;
        for (int u0 = 0; u0 < KS; u0 += 16) {
            float z[16];
            for (int u = 0; u < 16; ++u) {
                const int lj = k0 + u0 + u;
                z[u] = (valid && lj <= li) ? a.scale * sd[lj] + ci - sC[u0 + u] : -INFINITY;
            }
            process(z, 16, u0);
        }
    }
    // off-diagonal tiles, right to left
    const long long npairs = (long long)nblk * (nblk - 1) / 2;
    for (int J = I - 1; J >= 0; --J) {
        const TM *kh = static_cast<const TM *>(a.Khat) + ((long long)h * npairs + pair_index(I, J)) * BT * D;
        for (int k0 = 0; k0 < BT; k0 += KS) {
            __syncthreads();
            stage_rows<TM, D>(sK, D, kh + (long long)k0 * D, KS);
            stage_rows<T, D>(sV, D, V + (long long)(J * BT + k0) * D, KS);
            for (int u = threadIdx.x; u < KS; u += blockDim.x)
                sC[u] = a.c ? a.c[(long long)h * Lp + J * BT + k0 + u] : 0.f;
            __syncthreads();
            for (int u0 = 0; u0 < KS; u0 += 16) {
                float z[16];
                for (int u = 0; u < 16; ++u) {
                    const float *kr = sK + (u0 + u) * D;
                    float s = 0.f;
                    for (int e = 0; e < D; ++e) s = fmaf(sQ[e * QR + threadIdx.x], kr[e], s);
                    z[u] = valid ? a.scale * s + ci - sC[u0 + u] : -INFINITY;
                }
                process(z, 16, u0);
            }
        }
    }
    if (!valid) return;
    const float inv = 1.f / l;
    TO *out = static_cast<TO *>(a.out) + ((long long)h * L + gi) * D;
    for (int e = 0; e < D; ++e) out[e] = from_f<TO>(o[e] * inv);
    a.lse[(long long)h * L + gi] = m + __logf(l);
}

// ---------------------------------------------------------------------------
// Backward, query side: dQtil (off-diagonal pairs), dSd (diagonal tiles),
// row sums of dZ. grid (2*nblk, nh), QR threads.
// ---------------------------------------------------------------------------
template <typename T, typename TM, typename TO, int D>
__global__ void __launch_bounds__(QR) bwd_q_kernel(BwdArgs a)
{
    extern __shared__ float sm[];
    float *sQ = sm;                // [D][QR]
    float *sDO = sQ + D * QR;      // [D][QR]
    float *sK = sDO + D * QR;      // [KS][D]
    float *sV = sK + KS * D;       // [KS][D]
    float *sC = sV + KS * D;       // [KS]
    const int I = blockIdx.x / 2, half = blockIdx.x % 2, h = blockIdx.y;
    const int L = a.L, nblk = a.nblk, Lp = nblk * BT;
    const int li = half * QR + threadIdx.x;
    const int gi = I * BT + li;
    const bool valid = gi < L;
    const TM *qt = static_cast<const TM *>(a.Qt) + ((long long)h * Lp + gi) * D;
    const TO *dO = static_cast<const TO *>(a.dout) + ((long long)h * L + (valid ? gi : 0)) * D;
    for (int e = 0; e < D; ++e) {
        sQ[e * QR + threadIdx.x] = to_f(qt[e]);
        sDO[e * QR + threadIdx.x] = valid ? to_f(dO[e]) : 0.f;
    }
    const float ci = (a.c && valid) ? a.c[(long long)h * Lp + gi] : 0.f;
    const float lse = valid ? a.lse[(long long)h * L + gi] : 0.f;
    const float delta = valid ? a.delta[(long long)h * Lp + gi] : 0.f;
    float dq[D];
    for (int e = 0; e < D; ++e) dq[e] = 0.f;
    float rowsum = 0.f;
    const T *V = static_cast<const T *>(a.v) + (long long)h * L * D;
    // diagonal tile
    float *dsd = a.dSd + (((long long)h * nblk + I) * BT + li) * BT;
    const float *sd = a.Sd + (((long long)h * nblk + I) * BT + li) * BT;
    for (int k0 = 0; k0 < BT; k0 += KS) {
        __syncthreads();
        const int rows = min(KS, L - (I * BT + k0));
        stage_rows<T, D>(sV, D, V + (long long)(I * BT + k0) * D, rows);
        for (int u = threadIdx.x; u < KS; u += blockDim.x)
            sC[u] = a.c ? a.c[(long long)h * Lp + I * BT + k0 + u] : 0.f;
        __syncthreads();
        for (int u = 0; u < KS; ++u) {
            const int lj = k0 + u;
            float ds = 0.f;
            if (valid && lj <= li) {
                const float p = __expf(a.scale * sd[lj] + ci - sC[u] - lse);
                const float *vr = sV + u * D;
                float dp = 0.f;
                for (int e = 0; e < D; ++e) dp = fmaf(sDO[e * QR + threadIdx.x], vr[e], dp);
                const float dz = p * (dp - delta);
                rowsum += dz;
                ds = a.scale * dz;
            }
            dsd[lj] = ds;
        }
    }
    const long long npairs = (long long)nblk * (nblk - 1) / 2;
    for (int J = I - 1; J >= 0; --J) {
        const TM *kh = static_cast<const TM *>(a.Khat) + ((long long)h * npairs + pair_index(I, J)) * BT * D;
        for (int k0 = 0; k0 < BT; k0 += KS) {
            __syncthreads();
            stage_rows<TM, D>(sK, D, kh + (long long)k0 * D, KS);
            stage_rows<T, D>(sV, D, V + (long long)(J * BT + k0) * D, KS);
            for (int u = threadIdx.x; u < KS; u += blockDim.x)
                sC[u] = a.c ? a.c[(long long)h * Lp + J * BT + k0 + u] : 0.f;
            __syncthreads();
            if (!valid) continue;
            for (int u = 0; u < KS; ++u) {
                const float *kr = sK + u * D, *vr = sV + u * D;
                float s = 0.f, dp = 0.f;
                for (int e = 0; e < D; ++e) {
                    s = fmaf(sQ[e * QR + threadIdx.x], kr[e], s);
                    dp = fmaf(sDO[e * QR + threadIdx.x], vr[e], dp);
                }
                const float p = __expf(a.scale * s + ci - sC[u] - lse);
                const float dz = p * (dp - delta);
                rowsum += dz;
                const float ds = a.scale * dz;
                for (int e = 0; e < D; ++e) dq[e] = fmaf(ds, kr[e], dq[e]);
            }
        }
    }
    float *dqt = a.dQt + ((long long)h * Lp + gi) * D;
    for (int e = 0; e < D; ++e) dqt[e] = valid ? dq[e] : 0.f;
    if (a.rowsum) a.rowsum[(long long)h * Lp + gi] = valid ? rowsum : 0.f;
}

// ---------------------------------------------------------------------------
// Backward, key side: dV, the adjoint of the transport chain (-> dKtil),
// dP (atomically accumulated), column sums of dZ.
// grid (2*nblk, nh), QR threads; thread j = key row.
// ---------------------------------------------------------------------------
template <typename T, typename TM, typename TO, int D>
__global__ void __launch_bounds__(QR) bwd_k_kernel(BwdArgs a)
{
    extern __shared__ float sm[];
    float *sQ = sm;                    // [QR][D]   (query rows, broadcast)
    float *sDO = sQ + QR * D;          // [QR][D]
    float *sKh = sDO + QR * D;         // [QR][D+1] (own key rows)
    float *sVj = sKh + QR * (D + 1);   // [QR][D+1]
    float *sAb = sVj + QR * (D + 1);   // [QR][D+1]
    float *sP = sAb + QR * (D + 1);    // [D][D]
    float *sRow = sP + D * D;          // [3][QR]: lse, delta, c of query rows
    const int J = blockIdx.x / 2, half = blockIdx.x % 2, h = blockIdx.y;
    const int L = a.L, nblk = a.nblk, Lp = nblk * BT;
    const int lj = half * QR + threadIdx.x;
    const int gj = J * BT + lj;
    const bool valid = gj < L;
    const int t = threadIdx.x;
    float *kh = sKh + t * (D + 1), *vj = sVj + t * (D + 1), *ab = sAb + t * (D + 1);
    const T *V = static_cast<const T *>(a.v) + (long long)h * L * D;
    const TO *dOut = static_cast<const TO *>(a.dout) + (long long)h * L * D;
    for (int e = 0; e < D; ++e) {
        vj[e] = valid ? to_f(V[(long long)gj * D + e]) : 0.f;
        ab[e] = 0.f;
    }
    const float cj = (a.c && valid) ? a.c[(long long)h * Lp + gj] : 0.f;
    float dv[D];
    for (int e = 0; e < D; ++e) dv[e] = 0.f;
    float colsum = 0.f;
    const long long npairs = (long long)nblk * (nblk - 1) / 2;
    auto stage_queries = [&](int I, int q0) {
        const TM *qt = static_cast<const TM *>(a.Qt) + ((long long)h * Lp + I * BT + q0) * D;
        const int rows = min(QR, L - (I * BT + q0));
        for (int e = t; e < QR * D; e += blockDim.x) {
            const int r = e / D, c = e % D;
            sQ[e] = to_f(qt[(long long)r * D + c]);
            sDO[e] = r < rows ? to_f(dOut[(long long)(I * BT + q0 + r) * D + c]) : 0.f;
        }
        for (int r = t; r < QR; r += blockDim.x) {
            const int gi = I * BT + q0 + r;
            sRow[r] = gi < L ? a.lse[(long long)h * L + gi] : 0.f;
            sRow[QR + r] = gi < L ? a.delta[(long long)h * Lp + gi] : 0.f;
            sRow[2 * QR + r] = (a.c && gi < L) ? a.c[(long long)h * Lp + gi] : 0.f;
        }
    };
    for (int I = nblk - 1; I > J; --I) {
        __syncthreads();
        const TM *khat = static_cast<const TM *>(a.Khat) +
                        ((long long)h * npairs + pair_index(I, J)) * BT * D + (long long)lj * D;
        for (int e = 0; e < D; ++e) kh[e] = to_f(khat[e]);
        if (I + 1 < nblk) {
            // dP_I += Abar_{I+1}^T Khat_{J,I}   and   Abar <- Abar_{I+1} P_I
            const TM *p = static_cast<const TM *>(a.Pm) + ((long long)h * nblk + I) * D * D;
            for (int e = t; e < D * D; e += blockDim.x) sP[e] = to_f(p[e]);
            __syncthreads();
            float *dpm = a.dPm + ((long long)h * nblk + I) * D * D;
            for (int o = t; o < D * D; o += blockDim.x) {
                const int e = o / D, f = o % D;
                float s = 0.f;
                for (int r = 0; r < QR; ++r) s = fmaf(sAb[r * (D + 1) + e], sKh[r * (D + 1) + f], s);
                atomicAdd(dpm + o, s);
            }
            __syncthreads();
            float nab[D];
            for (int e = 0; e < D; ++e) {
                float s = 0.f;
                for (int f = 0; f < D; ++f) s = fmaf(ab[f], sP[f * D + e], s);
                nab[e] = s;
            }
            for (int e = 0; e < D; ++e) ab[e] = nab[e];
        }
        for (int q0 = 0; q0 < BT; q0 += QR) {
            __syncthreads();
            stage_queries(I, q0);
            __syncthreads();
            const int rows = min(QR, L - (I * BT + q0));
            if (!valid) continue;
            for (int r = 0; r < rows; ++r) {
                const float *qr = sQ + r * D, *dor = sDO + r * D;
                float s = 0.f, dp = 0.f;
                for (int e = 0; e < D; ++e) {
                    s = fmaf(qr[e], kh[e], s);
                    dp = fmaf(dor[e], vj[e], dp);
                }
                const float p = __expf(a.scale * s + sRow[2 * QR + r] - cj - sRow[r]);
                const float dz = p * (dp - sRow[QR + r]);
                colsum += dz;
                const float ds = a.scale * dz;
                for (int e = 0; e < D; ++e) {
                    dv[e] = fmaf(p, dor[e], dv[e]);
                    ab[e] = fmaf(ds, qr[e], ab[e]);
                }
            }
        }
    }
    // the chain's adjoint at its start is the gradient of Ktil
    float *dkt = a.dKt + ((long long)h * Lp + gj) * D;
    for (int e = 0; e < D; ++e) dkt[e] = valid ? ab[e] : 0.f;
    // diagonal tile: queries i >= j of tile J
    const float *sd = a.Sd + ((long long)h * nblk + J) * BT * BT;
    for (int q0 = 0; q0 < BT; q0 += QR) {
        __syncthreads();
        stage_queries(J, q0);
        __syncthreads();
        const int rows = min(QR, L - (J * BT + q0));
        if (!valid) continue;
        for (int r = 0; r < rows; ++r) {
            const int li = q0 + r;
            if (li < lj) continue;
            const float *dor = sDO + r * D;
            float dp = 0.f;
            for (int e = 0; e < D; ++e) dp = fmaf(dor[e], vj[e], dp);
            const float p = __expf(a.scale * sd[(long long)li * BT + lj] + sRow[2 * QR + r] - cj - sRow[r]);
            const float dz = p * (dp - sRow[QR + r]);
            colsum += dz;
            for (int e = 0; e < D; ++e) dv[e] = fmaf(p, dor[e], dv[e]);
        }
    }
    if (!valid) return;
    TO *dvo = static_cast<TO *>(a.dv) + ((long long)h * L + gj) * D;
    for (int e = 0; e < D; ++e) dvo[e] = from_f<TO>(dv[e]);
    if (a.colsum) a.colsum[(long long)h * Lp + gj] = colsum;
}

// delta_i = dO_i . O_i, one warp per row (coalesced row reads)
template <typename T, int D>
__global__ void delta_kernel(const T *out, const T *dout, float *delta, int L, int Lp, int nh)
{
    const int lane = threadIdx.x % 32;
    const long long n = (long long)nh * Lp;
    const long long warps = (long long)gridDim.x * (blockDim.x / 32);
    for (long long x = blockIdx.x * (long long)(blockDim.x / 32) + threadIdx.x / 32; x < n; x += warps) {
        const int h = (int)(x / Lp), i = (int)(x % Lp);
        float s = 0.f;
        if (i < L) {
            const T *o = out + ((long long)h * L + i) * D, *g = dout + ((long long)h * L + i) * D;
            for (int e = lane; e < D; e += 32) s = fmaf(to_f(o[e]), to_f(g[e]), s);
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
        if (lane == 0) delta[x] = s;
    }
}

// The same as delta_kernel with 16-byte loads (out and dout 16-byte aligned): a
// row is D / VE lanes of VE elements, a warp takes 32 / (D / VE) rows per step,
// and a reduction over the row's lanes.
template <typename T, int D>
__global__ void delta_vec_kernel(const T *out, const T *dout, float *delta, int L, int Lp, int nh)
{
    constexpr int VE = 16 / (int)sizeof(T), LPR = D / VE, RPW = 32 / LPR;
    const int lane = threadIdx.x % 32, sub = lane % LPR;
    const long long n = (long long)nh * Lp;
    const long long warps = (long long)gridDim.x * (blockDim.x / 32);
    for (long long x0 = (blockIdx.x * (long long)(blockDim.x / 32) + threadIdx.x / 32) * RPW; x0 < n;
         x0 += warps * RPW) {
        const long long x = x0 + lane / LPR;
        float s = 0.f;
        if (x < n) {
            const int h = (int)(x / Lp), i = (int)(x % Lp);
            if (i < L) {
                const long long off = ((long long)h * L + i) * D + sub * VE;
                const uint4 uo = *reinterpret_cast<const uint4 *>(out + off);
                const uint4 ug = *reinterpret_cast<const uint4 *>(dout + off);
                const T *o = reinterpret_cast<const T *>(&uo), *g = reinterpret_cast<const T *>(&ug);
#pragma unroll
                for (int e = 0; e < VE; ++e) s = fmaf(to_f(o[e]), to_f(g[e]), s);
            }
        }
#pragma unroll
        for (int m = LPR / 2; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
        if (sub == 0 && x < n) delta[x] = s;
    }
}

// c_t = sum_{s<=t} log f_s (fp64 running sum), padded rows repeat the last value
// Block-wide inclusive scan of one double per thread (blockDim.x = GATE_NT).
constexpr int GATE_NT = 1024;

__device__ double block_inclusive_scan(double v)
{
    __shared__ double sh[GATE_NT];
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < GATE_NT; o <<= 1) {
        const double add = threadIdx.x >= (unsigned)o ? sh[threadIdx.x - o] : 0.0;
        __syncthreads();
        sh[threadIdx.x] += add;
        __syncthreads();
    }
    return sh[threadIdx.x];
}

// c_t = sum_{s<=t} log f_s (0 past L), accumulated in fp64: one block per head, each
// thread a contiguous chunk of positions (chunk sums, a block scan of them, the chunk).
__global__ void __launch_bounds__(GATE_NT) gate_prefix_kernel(const float *logf, float *c, int L, int Lp)
{
    const long long h = blockIdx.x;
    const int n = (Lp + GATE_NT - 1) / GATE_NT, t0 = threadIdx.x * n, t1 = min(t0 + n, Lp);
    const float *lf = logf + h * L;
    double s = 0.0;
    for (int t = t0; t < t1 && t < L; ++t) s += lf[t];
    double acc = block_inclusive_scan(s) - s;
    for (int t = t0; t < t1; ++t) {
        if (t < L) acc += lf[t];
        c[h * Lp + t] = (float)acc;
    }
}

// dlogf_s = sum_{t>=s} (rowsum_t - colsum_t), in fp64: one block per head, thread k the
// k-th chunk from the end.
__global__ void __launch_bounds__(GATE_NT) gate_grad_kernel(const float *rowsum, const float *colsum,
                                                           float *dlogf, int L, int Lp)
{
    const long long h = blockIdx.x;
    const int n = (L + GATE_NT - 1) / GATE_NT;
    const int t1 = L - threadIdx.x * n, t0 = max(t1 - n, 0);  // chunk [t0, t1), counted from the end
    const float *rs = rowsum + h * Lp, *cs = colsum + h * Lp;
    double s = 0.0;
    for (int t = t0; t < t1; ++t) s += (double)rs[t] - (double)cs[t];
    double acc = block_inclusive_scan(s) - s;
    for (int t = t1 - 1; t >= t0; --t) {
        acc += (double)rs[t] - (double)cs[t];
        dlogf[h * L + t] = (float)acc;
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define CK(x)                             \
    do {                                  \
        cudaError_t e_ = (x);             \
        if (e_ != cudaSuccess) return e_; \
    } while (0)

template <typename T, int D>
cudaError_t run_chain(const ChainArgs &c, cudaStream_t st)
{
    if (c.nblk < 2) return cudaSuccess;
    const size_t smem = (D * D + BT * (D + 1)) * sizeof(float);
    CK(set_smem(chain_kernel<T, D>, smem));
    chain_kernel<T, D><<<dim3(c.nblk - 1, c.nh), BT, smem, st>>>(
        static_cast<const T *>(c.Kt), static_cast<const T *>(c.Pm), static_cast<T *>(c.Khat), c.nblk);
    count_launches();
    return cudaGetLastError();
}

template <typename T, typename TM, typename TO, int D>
cudaError_t run_fwd(const FwdArgs &a, cudaStream_t st)
{
    const size_t smem = (D * QR + 2 * KS * D + KS) * sizeof(float);
    CK(set_smem(fwd_kernel<T, TM, TO, D>, smem));
    fwd_kernel<T, TM, TO, D><<<dim3(2 * a.nblk, a.nh), QR, smem, st>>>(a);
    count_launches();
    return cudaGetLastError();
}

template <typename T, typename TM, typename TO, int D>
cudaError_t run_bwd(const BwdArgs &a, cudaStream_t st)
{
    const int Lp = a.nblk * BT;
    delta_kernel<TO, D><<<1184, 256, 0, st>>>(static_cast<const TO *>(a.out),
                                             static_cast<const TO *>(a.dout), a.delta, a.L, Lp, a.nh);
    count_launches();
    CK(cudaGetLastError());
    const size_t smq = (2 * D * QR + 2 * KS * D + KS) * sizeof(float);
    CK(set_smem(bwd_q_kernel<T, TM, TO, D>, smq));
    {
        Stage s_q("attn_bwd_q", st);
        bwd_q_kernel<T, TM, TO, D><<<dim3(2 * a.nblk, a.nh), QR, smq, st>>>(a);
        count_launches();
    }
    CK(cudaGetLastError());
    const size_t smk = (2 * QR * D + 3 * QR * (D + 1) + D * D + 3 * QR) * sizeof(float);
    CK(set_smem(bwd_k_kernel<T, TM, TO, D>, smk));
    {
        Stage s_k("attn_bwd_k", st);
        bwd_k_kernel<T, TM, TO, D><<<dim3(2 * a.nblk, a.nh), QR, smk, st>>>(a);
        count_launches();
    }
    return cudaGetLastError();
}

template <int D, typename F>
cudaError_t by_types(Types t, F &&f)
{
    using DD = std::integral_constant<int, D>;
    if (t.in == F32) return f(float(), float(), float(), DD());
    if (t.out == BF16) return f(bf16(), f16(), bf16(), DD());
    return f(bf16(), f16(), float(), DD());
}

template <typename F>
cudaError_t dispatch(Types t, int d, F &&f)
{
    switch (d) {
    case 16: return by_types<16>(t, f);
    case 32: return by_types<32>(t, f);
    case 64: return by_types<64>(t, f);
    case 128: return by_types<128>(t, f);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t chain_simt(const ChainArgs &c, Types t, int d, cudaStream_t st)
{
    return dispatch(t, d, [&](auto, auto i, auto, auto dd) {
        return run_chain<decltype(i), decltype(dd)::value>(c, st);
    });
}

cudaError_t attn_fwd_simt(const FwdArgs &a, Types t, int d, cudaStream_t st)
{
    return dispatch(t, d, [&](auto x, auto i, auto o, auto dd) {
        return run_fwd<decltype(x), decltype(i), decltype(o), decltype(dd)::value>(a, st);
    });
}

cudaError_t attn_bwd_simt(const BwdArgs &a, Types t, int d, cudaStream_t st)
{
    return dispatch(t, d, [&](auto x, auto i, auto o, auto dd) {
        return run_bwd<decltype(x), decltype(i), decltype(o), decltype(dd)::value>(a, st);
    });
}

cudaError_t compute_delta(const BwdArgs &a, Types t, int d, cudaStream_t st)
{
    const bool vec = ((reinterpret_cast<uintptr_t>(a.out) | reinterpret_cast<uintptr_t>(a.dout)) & 15u) == 0;
    return dispatch(t, d, [&](auto, auto, auto o, auto dd) {
        using TO = decltype(o);
        constexpr int DD = decltype(dd)::value;
        if (vec && DD * (int)sizeof(TO) >= 32)
            delta_vec_kernel<TO, DD><<<1184, 256, 0, st>>>(static_cast<const TO *>(a.out),
                                                           static_cast<const TO *>(a.dout), a.delta,
                                                           a.L, a.nblk * BT, a.nh);
        else
            delta_kernel<TO, DD><<<1184, 256, 0, st>>>(static_cast<const TO *>(a.out),
                                                       static_cast<const TO *>(a.dout), a.delta, a.L,
                                                       a.nblk * BT, a.nh);
        count_launches();
        return cudaGetLastError();
    });
}

cudaError_t gate_prefix(const float *logf, float *c, int L, int Lp, int nh, cudaStream_t st)
{
    gate_prefix_kernel<<<nh, GATE_NT, 0, st>>>(logf, c, L, Lp);
    count_launches();
    return cudaGetLastError();
}

cudaError_t gate_grad(const float *rowsum, const float *colsum, float *dlogf, int L, int Lp, int nh,
                      cudaStream_t st)
{
    gate_grad_kernel<<<nh, GATE_NT, 0, st>>>(rowsum, colsum, dlogf, L, Lp);
    count_launches();
    return cudaGetLastError();
}

}  // namespace path
