// common.cuh -- device helpers shared by the kernels of libacl (sm_100a).
//
// Thin wrappers over PTX: cp.async 16-byte copies (zero-fill for empty slots),
// ldmatrix / movmatrix 8x8 b16 fragment moves and the m16n8k16 bf16 tensor-core
// product with fp32 accumulation.  Fragment layouts (thread lane = 4*g + t):
//   A (16x16, row-major): reg0 = A[g][2t..2t+1],   reg1 = A[g+8][2t..2t+1],
//                         reg2 = A[g][2t+8..2t+9], reg3 = A[g+8][2t+8..2t+9]
//   B (16x8, k-major):    reg0 = B[2t..2t+1][g],   reg1 = B[2t+8..2t+9][g]
//   C (16x8, fp32):       c0,c1 = C[g][2t..2t+1],  c2,c3 = C[g+8][2t..2t+1]
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace acl {

typedef __nv_bfloat16 bf16;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device-side consistency checks of the check build (compiled with -DACL_DEVICE_CHECKS):
// ACL_DEVICE_CHECK(cond) records a failed condition in a flag word of the translation unit,
// which acl_device_check reads (ACL_ERR_DEVICE_CHECK) and clears.  The kernels handle the
// condition as the regular build does (an out-of-range token id is an empty slot); the check
// build only reports it.  In the regular build the macro compiles to nothing.
#ifdef ACL_DEVICE_CHECKS
static __device__ unsigned int g_check_flags;
#define ACL_DEVICE_CHECK(cond)                                       \
    do {                                                             \
        if (!(cond)) atomicOr(&::acl::g_check_flags, 1u);            \
    } while (0)
#define ACL_CHECK_READER(name)                                                      \
    cudaError_t name(unsigned int* flags) {                                         \
        cudaError_t e = cudaMemcpyFromSymbol(flags, ::acl::g_check_flags, sizeof(unsigned int)); \
        if (e != cudaSuccess) return e;                                             \
        const unsigned int zero = 0u;                                               \
        return cudaMemcpyToSymbol(::acl::g_check_flags, &zero, sizeof(unsigned int)); \
    }
#else
#define ACL_DEVICE_CHECK(cond) ((void)0)
#define ACL_CHECK_READER(name)                      \
    cudaError_t name(unsigned int* flags) {         \
        *flags = 0u;                                \
        return cudaSuccess;                         \
    }
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; when !valid nothing is read and the 16 bytes are zeroed.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}
// 8-byte global->shared copy (L1-allocating form); when !valid the 8 bytes are zeroed.
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, bool valid) {
    int n = valid ? 8 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(dst), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Transpose of an 8x8 b16 matrix held one 32-bit pair per lane (row = lane/4).
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

// c += A(16x16 bf16) * B(16x8 bf16), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two floats -> packed bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of 16-byte chunk `ch` (0..3) of row `row` in a 64-byte-row tile, XOR-swizzled
// so that the 8 rows an ldmatrix reads fall in 8 distinct bank groups.
__device__ __forceinline__ uint32_t tile64_off(int row, int ch) {
    return static_cast<uint32_t>(row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
}

// Read-only 16-byte global load through the non-coherent path.
__device__ __forceinline__ uint4 ldg16(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Grid cell of a coordinate on an axis of n cells: clamp(floor(v), 0, n - 1); a value that
// is not >= 0 (negative or NaN) maps to 0.  Used for queries (gather) and tokens (order).
__device__ __forceinline__ int quantise(float v, int n) {
    if (!(v >= 0.f)) return 0;
    if (v >= static_cast<float>(n)) return n - 1;
    const int i = static_cast<int>(v);
    return i > n - 1 ? n - 1 : i;
}

}  // namespace acl
