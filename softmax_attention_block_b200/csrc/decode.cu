// Decode step: fused in-place key update + one-query attention over the
// cache, split over chunks of rows (Paper-Notes "训练策略", inference
// paragraph: cached keys are updated in place by H_t, after which decoding
// is plain softmax attention). With the forget gate (Paper-Notes "PaTH-FoX
// 扩展": the logit gains c_t - c_j), each cached key also carries that bias,
// updated in place by the same pass: g_j += log f_t, and the new key's is 0.
//
// Pass 1 (decode_chunk_kernel): each CTA streams DECODE_CHUNK cached rows of
// one head. A group of d/V lanes owns one row at a time (V elements of 16
// bytes per lane): it reads k and v once, writes the updated k once, and keeps
// a running (max, sum, acc) of the softmax. Pass 2 (decode_combine_kernel)
// merges the chunks with the new key, which it also appends to the caches.
#include <mutex>

#include "attn.cuh"
#include "runtime.cuh"

namespace path {

namespace {

template <typename T>
struct Vec {
    static constexpr int N = 16 / sizeof(T);
};

template <typename T>
__device__ __forceinline__ void unpack(const uint4 &u, float *f)
{
    if constexpr (sizeof(T) == 4) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    } else {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack(const float *f)
{
    uint4 u;
    if constexpr (sizeof(T) == 4) {
        u.x = __float_as_uint(f[0]);
        u.y = __float_as_uint(f[1]);
        u.z = __float_as_uint(f[2]);
        u.w = __float_as_uint(f[3]);
    } else {
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    }
    return u;
}

// round-trip through the storage type (what the cache will hold)
template <typename T>
__device__ __forceinline__ void round_to(float *f)
{
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = __bfloat162float(__float2bfloat16_rn(f[i]));
    }
}

template <int LPR>
__device__ __forceinline__ float group_sum(float x)
{
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

constexpr int THREADS = 256;
constexpr int UNROLL = 8;  // rows in flight per row group (loads issued before the math)

template <typename T, int D, bool GATE, int CHUNK = DECODE_CHUNK>
__global__ void __launch_bounds__(THREADS) decode_chunk_kernel(DecodeArgs a, int nchunk)
{
    constexpr int V = Vec<T>::N;        // elements per 16-byte vector
    constexpr int LPR = D / V;          // lanes per row
    constexpr int G = THREADS / LPR;    // row groups per CTA
    __shared__ float s_m[G], s_l[G];
    __shared__ float s_acc[G][D];
    const int chunk = blockIdx.x, h = blockIdx.y;
    const int lane_in_row = threadIdx.x % LPR, g = threadIdx.x / LPR;
    const int r0 = chunk * CHUNK;
    const int r1 = min(a.n, r0 + CHUNK);
    float w[V], q[V];
    unpack<T>(reinterpret_cast<const uint4 *>(static_cast<const T *>(a.w) + (long long)h * D)[lane_in_row], w);
    unpack<T>(reinterpret_cast<const uint4 *>(static_cast<const T *>(a.q) + (long long)h * D)[lane_in_row], q);
    const float beta = a.beta[h];
    const float lf = GATE ? a.log_f[h] : 0.f;
    float *gc = GATE ? a.g_cache + (long long)h * a.capacity : nullptr;
    uint4 *K = reinterpret_cast<uint4 *>(static_cast<T *>(a.k_cache) + (long long)h * a.capacity * D);
    const uint4 *Vc = reinterpret_cast<const uint4 *>(static_cast<const T *>(a.v_cache) + (long long)h * a.capacity * D);
    float m = -INFINITY, l = 0.f, acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    // waves of G * UNROLL rows: the loop bound is uniform across the CTA, so
    // every lane reaches every group shuffle; rows past the chunk are masked.
    for (int rb = r0; rb < r1; rb += G * UNROLL) {
        uint4 kv[UNROLL], vv[UNROLL];
        float gv[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int r = rb + u * G + g;
            gv[u] = 0.f;
            if (r < r1) {
                kv[u] = K[(long long)r * LPR + lane_in_row];
                vv[u] = Vc[(long long)r * LPR + lane_in_row];
                if (GATE) gv[u] = gc[r];
            } else {
                kv[u] = make_uint4(0u, 0u, 0u, 0u);
                vv[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int r = rb + u * G + g;
            const bool valid = r < r1;
            float k[V], v[V];
            unpack<T>(kv[u], k);
            unpack<T>(vv[u], v);
            float wk = 0.f;
#pragma unroll
            for (int i = 0; i < V; ++i) wk = fmaf(w[i], k[i], wk);
            wk = group_sum<LPR>(wk);
            const float coef = beta * wk;
#pragma unroll
            for (int i = 0; i < V; ++i) k[i] = fmaf(-coef, w[i], k[i]);
            if (valid) K[(long long)r * LPR + lane_in_row] = pack<T>(k);
            round_to<T>(k);
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < V; ++i) s = fmaf(q[i], k[i], s);
            s = group_sum<LPR>(s);
            float bias = 0.f;
            if (GATE) {
                bias = gv[u] + lf;
                if (valid && lane_in_row == 0) gc[r] = bias;
            }
            if (valid) {
                const float z = fmaf(a.scale, s, bias);
                const float mn = fmaxf(m, z);
                const float corr = __expf(m - mn);
                const float p = __expf(z - mn);
                l = fmaf(l, corr, p);
#pragma unroll
                for (int i = 0; i < V; ++i) acc[i] = fmaf(acc[i], corr, p * v[i]);
                m = mn;
            }
        }
    }
    // merge the row groups of this CTA
    if (lane_in_row == 0) {
        s_m[g] = m;
        s_l[g] = l;
    }
#pragma unroll
    for (int i = 0; i < V; ++i) s_acc[g][lane_in_row * V + i] = acc[i];
    __syncthreads();
    float *part = a.partial + ((long long)h * nchunk + chunk) * (D + 2);
    for (int e = threadIdx.x; e < D; e += THREADS) {
        float M = -INFINITY;
        for (int j = 0; j < G; ++j) M = fmaxf(M, s_m[j]);
        float Ls = 0.f, A = 0.f;
        for (int j = 0; j < G; ++j) {
            const float f = s_m[j] == -INFINITY ? 0.f : __expf(s_m[j] - M);
            Ls = fmaf(s_l[j], f, Ls);
            A = fmaf(s_acc[j][e], f, A);
        }
        part[2 + e] = A;
        if (e == 0) {
            part[0] = M;
            part[1] = Ls;
        }
    }
}

template <typename T, int D>
__global__ void decode_combine_kernel(DecodeArgs a, int nchunk)
{
    const int h = blockIdx.x, e = threadIdx.x;  // D threads
    __shared__ float red[D];
    __shared__ float s_z;
    const T *q = static_cast<const T *>(a.q) + (long long)h * D;
    const T *kn = static_cast<const T *>(a.k_new) + (long long)h * D;
    const T *vn = static_cast<const T *>(a.v_new) + (long long)h * D;
    red[e] = to_f(q[e]) * to_f(kn[e]);
    __syncthreads();
    if (e == 0) {
        float s = 0.f;
        for (int i = 0; i < D; ++i) s += red[i];
        s_z = a.scale * s;
    }
    __syncthreads();
    const float zn = s_z;
    float M = zn;
    for (int c = 0; c < nchunk; ++c) M = fmaxf(M, a.partial[((long long)h * nchunk + c) * (D + 2)]);
    float Ls = __expf(zn - M), A = Ls * to_f(vn[e]);
    for (int c = 0; c < nchunk; ++c) {
        const float *p = a.partial + ((long long)h * nchunk + c) * (D + 2);
        if (p[0] == -INFINITY) continue;
        const float f = __expf(p[0] - M);
        Ls = fmaf(p[1], f, Ls);
        A = fmaf(p[2 + e], f, A);
    }
    static_cast<T *>(a.out)[(long long)h * D + e] = from_f<T>(A / Ls);
    // append the new key / value untransformed
    const long long row = ((long long)h * a.capacity + a.n) * D + e;
    static_cast<T *>(a.k_cache)[row] = kn[e];
    static_cast<T *>(a.v_cache)[row] = vn[e];
    if (a.g_cache && e == 0) a.g_cache[(long long)h * a.capacity + a.n] = 0.f;
}

template <typename T, int D, int CHUNK>
void launch_chunks(const DecodeArgs &a, int nchunk, cudaStream_t st)
{
    if (a.g_cache)
        decode_chunk_kernel<T, D, true, CHUNK><<<dim3(nchunk, a.nh), THREADS, 0, st>>>(a, nchunk);
    else
        decode_chunk_kernel<T, D, false, CHUNK><<<dim3(nchunk, a.nh), THREADS, 0, st>>>(a, nchunk);
}

template <typename T, int D>
cudaError_t run(const DecodeArgs &a, cudaStream_t st)
{
    const int nchunk = ceil_div(a.n, DECODE_CHUNK);
    if (nchunk > 0) {
        Stage s("decode_chunks", st);
        launch_chunks<T, D, DECODE_CHUNK>(a, nchunk, st);
        count_launches();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    decode_combine_kernel<T, D><<<a.nh, D, 0, st>>>(a, nchunk);
    count_launches();
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the chunk partials live in a fixed device array.
// ---------------------------------------------------------------------------
template <typename T, int D, int CHUNK>
cudaError_t run_fixed(const DecodeArgs &a, cudaStream_t st)
{
    const int nchunk = ceil_div(a.n, CHUNK);
    if (nchunk > 0) {
        launch_chunks<T, D, CHUNK>(a, nchunk, st);
        count_launches();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    decode_combine_kernel<T, D><<<a.nh, D, 0, st>>>(a, nchunk);
    count_launches();
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t run_chunked(const DecodeArgs &a, int chunk, cudaStream_t st)
{
    switch (chunk) {
    case 256: return run_fixed<T, D, 256>(a, st);
    case 1024: return run_fixed<T, D, 1024>(a, st);
    case 4096: return run_fixed<T, D, 4096>(a, st);
    default: return run_fixed<T, D, 16384>(a, st);
    }
}

}  // namespace

// Scratch of path_decode_step_noalloc: NOALLOC_SCRATCH_FLOATS floats (4 MiB)
// in every GPU that loads the library, held until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[NOALLOC_SCRATCH_FLOATS];

int noalloc_chunk_rows(int nh, int n, int d)
{
    static const int sizes[] = {256, 1024, 4096, 16384};
    for (int c : sizes) {
        const long long need = (long long)nh * ceil_div(n > 0 ? n : 1, c) * (d + 2);
        if (need <= (long long)NOALLOC_SCRATCH_FLOATS) return c;
    }
    return 0;
}

cudaError_t noalloc_scratch(float **ptr)
{
    // cudaGetSymbolAddress once per device, with that device current; the
    // array's name in host code is only a host-side stand-in for it.
    static std::mutex mu;
    static float *cache[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        cache[dev] = static_cast<float *>(p);
    }
    *ptr = cache[dev];
    return cudaSuccess;
}

cudaError_t decode_step_noalloc(const DecodeArgs &a, int dt, int d, int chunk, cudaStream_t st)
{
    if (d == 64) return dt == F32 ? run_chunked<float, 64>(a, chunk, st) : run_chunked<bf16, 64>(a, chunk, st);
    if (d == 128) return dt == F32 ? run_chunked<float, 128>(a, chunk, st) : run_chunked<bf16, 128>(a, chunk, st);
    return cudaErrorInvalidValue;
}

cudaError_t decode_step(const DecodeArgs &a, int dt, int d, cudaStream_t st)
{
    if (d == 64) return dt == F32 ? run<float, 64>(a, st) : run<bf16, 64>(a, st);
    if (d == 128) return dt == F32 ? run<float, 128>(a, st) : run<bf16, 128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace path
