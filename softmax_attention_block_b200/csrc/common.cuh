// Shared device/host helpers of the PaTH attention library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/path_attn.h"

namespace path {

// Attention tile = UT block: 128 positions. Query tiles, key tiles and the
// blocks of the per-block UT transform all use this size.
constexpr int BT = 128;

typedef __nv_bfloat16 bf16;
typedef __half f16;

// element types of device buffers
enum DType { F32 = 0, BF16 = 1, F16 = 2 };

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(f16 x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ f16 from_f<f16>(float x) { return __float2half_rn(x); }

__device__ __forceinline__ float load_as_f(const void *p, int dt, long long i)
{
    if (dt == F32) return static_cast<const float *>(p)[i];
    if (dt == BF16) return __bfloat162float(static_cast<const bf16 *>(p)[i]);
    return __half2float(static_cast<const f16 *>(p)[i]);
}

__device__ __forceinline__ void store_from_f(void *p, int dt, long long i, float x)
{
    if (dt == F32)
        static_cast<float *>(p)[i] = x;
    else if (dt == BF16)
        static_cast<bf16 *>(p)[i] = __float2bfloat16_rn(x);
    else
        static_cast<f16 *>(p)[i] = __float2half_rn(x);
}

inline size_t dtype_size(int dt) { return dt == F32 ? 4 : 2; }

// The three element types one call works with:
//   in  - q, k, v, w (and the decode caches)
//   mid - the computed boundary-adjusted queries/keys, block products and
//         transported keys (fp16 on the bf16 paths: same tensor-core rate as
//         bf16, three more mantissa bits)
//   out - out, dout and the gradients dq, dk, dv, dw
struct Types {
    int in, mid, out;
};

inline Types types_of(path_dtype dt)
{
    if (dt == PATH_F32) return {F32, F32, F32};
    if (dt == PATH_BF16) return {BF16, F16, BF16};
    return {BF16, F16, F32};  // PATH_BF16_F32OUT
}

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over the caller's workspace (256-byte aligned slices).
struct Carver {
    char *base;
    size_t off = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <typename T>
    T *take(size_t count)
    {
        off = align_up(off, 256);
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
    size_t bytes() const { return align_up(off, 256); }
};

// ---------------------------------------------------------------------------
// Batched small GEMM ("tiny BLAS") over the (head, block) grid of the UT
// transform. A batch item z = h * nblk + blk. Every operand names its own
// strides so that user tensors ([heads, L, d]) and scratch ([heads, nblk, ..])
// can be mixed.
// ---------------------------------------------------------------------------
enum Mask { MASK_NONE = 0, MASK_LOWER = 1, MASK_STRICT_LOWER = 2 };

struct Operand {
    const void *p = nullptr;
    int dt = F32;
    long long sh = 0;  // stride between heads (elements)
    long long sb = 0;  // stride between blocks (elements)
    int ld = 0;        // leading dimension of the stored matrix
    int trans = 0;     // use the transpose of the stored matrix
    int mask = 0;      // Mask, applied on STORED (row, col) indices
    int seq = -1;      // if >= 0: stored row r of block blk is zero when blk*BT + r >= seq
};

struct Term {
    Operand a, b;
    float alpha = 1.f;
};

struct GemmArgs {
    Term t[3];
    int nterms = 0;
    int M = 0, N = 0, K = 0;
    Operand addend;          // optional: C += gamma * addend (addend.p may be null)
    float gamma = 0.f;
    int add_identity = 0;    // C += I
    const float *rowscale = nullptr;  // optional per-output-row factor (applied to the product sum)
    long long rs_sh = 0, rs_sb = 0;
    int rs_seq = -1;         // rowscale entries at seq rows >= rs_seq read as 0
    int outmask = 0;         // Mask on output (r, c): masked elements are written as 0
    void *c = nullptr;
    int cdt = F32;
    long long csh = 0, csb = 0;
    int ldc = 0;
    int c_seq = -1;          // if >= 0: output rows with blk*BT + r >= c_seq are not written
    int nblk = 1;
    int batch = 1;           // number of batch items (heads * nblk)
    int *err = nullptr;      // device error word (tensor-core version: a wait that gave up)
};

// Launches the batched GEMM on `stream` (fp32 on CUDA cores). Returns cudaGetLastError().
cudaError_t gemm_batched(const GemmArgs &g, cudaStream_t stream);
// The same product on the tensor cores in TF32 (gemm_tc.cu), for M, N, K <= 128,
// multiples of 4, operands addressable four elements at a time.
bool gemm_tc_supported(const GemmArgs &g);
cudaError_t gemm_batched_tc(const GemmArgs &g, cudaStream_t stream);

}  // namespace path
