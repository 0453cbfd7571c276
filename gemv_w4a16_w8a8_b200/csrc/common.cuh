// Shared device helpers and the internal launch interface of the qgemm library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qgemm.h"

namespace qg {

// ------------------------------------------------------------------------------------------
// Problem description handed from the API layer to the kernel launchers.
// ------------------------------------------------------------------------------------------
struct Problem {
    int op;
    const void *A;
    const void *W;
    const void *scales;
    const void *zeros;
    void *C;
    int M, N, K;
    int gs;        // effective group size (K when the caller passed -1 / 0)
    int has_zero;
    int interleaved = 0;   // 1 = the interleaved weight layout (W4A16: nibbles hold codes
                           // 0,2,4,6,1,3,5,7; W2A8: fields hold 0,4,1,5,2,6,3,7, 8,12,...)
    int sms = 148;         // multiprocessors of the device (persistent grids)
    const float *mult = nullptr;   // W8A8: per-channel multiplier -> int8 output (else int32)
};

// int8 requantisation of an exact int32 accumulator: clamp(rint(float(v) * m), -128, 127),
// every step a correctly rounded binary32 operation.
__device__ __forceinline__ int8_t requant_i8(int v, float m)
{
    const float r = rintf(__fmul_rn(__int2float_rn(v), m));
    return (int8_t)(int)fminf(fmaxf(r, -128.0f), 127.0f);
}

// Launchers return cudaGetLastError() after queueing their kernels on `stream`.
cudaError_t launch_gemv_w4a16(const Problem &p, const qgemm_config_t &cfg, cudaStream_t stream);
// ws_part / ws_count non-null: deterministic split-K through an fp32 workspace (see the
// kernel); null: plain store or red.global.add into a zeroed C.
cudaError_t launch_gemv_w4a16_tma(const Problem &p, const qgemm_config_t &cfg, unsigned int *err,
                                  cudaStream_t stream, float *ws_part = nullptr,
                                  unsigned int *ws_count = nullptr);
// Arrival counters the deterministic split-K needs (one per output tile of this config).
size_t gemv_w4a16_ws_tiles(const Problem &p, const qgemm_config_t &cfg);
// Persistent stream-K W4A16 kernel (path QG_PATH_STREAM); C must be zeroed first.
cudaError_t launch_gemv_w4a16_stream(const Problem &p, const qgemm_config_t &cfg,
                                     unsigned int *err, cudaStream_t stream);
// W4A16 for 1..8 tokens on the packed fp16 FMA pipe (config: path GEMV, bn = 2).
cudaError_t launch_gemv_w4a16_h2(const Problem &p, const qgemm_config_t &cfg, unsigned int *err,
                                 cudaStream_t stream);
int gemv_w4a16_h2_tokens(int M);
cudaError_t launch_gemv_w2a8_tma(const Problem &p, const qgemm_config_t &cfg, unsigned int *err,
                                 cudaStream_t stream);
cudaError_t launch_gemv_int(const Problem &p, const qgemm_config_t &cfg, cudaStream_t stream);
// A kernel whose bounded wait can never be satisfied: it gives up after limit_ns and raises *err.
cudaError_t launch_wait_selftest(unsigned int *err, unsigned long long limit_ns,
                                 cudaStream_t stream);
cudaError_t launch_pack_int4(const uint8_t *codes, uint32_t *packed, int N, int K,
                             cudaStream_t stream);
cudaError_t launch_pack_int4_interleaved(const uint8_t *codes, uint32_t *packed, int N, int K,
                                         cudaStream_t stream);
// Round-to-nearest int4 quantisation (group size 32, 64, 128 or a multiple of 256 dividing K).
cudaError_t launch_rtn_int4(const __half *W, uint32_t *Wq, __half *S, __half *Z, int N, int K,
                            int gs, cudaStream_t stream);
cudaError_t launch_pack_int2(const int8_t *vals, uint32_t *packed, int N, int K,
                             cudaStream_t stream);
cudaError_t launch_pack_int2_interleaved(const int8_t *vals, uint32_t *packed, int N, int K,
                                         cudaStream_t stream);
cudaError_t launch_tc(const Problem &p, const qgemm_config_t &cfg, unsigned int *err_word,
                      cudaStream_t stream);

// Whether a configuration can run the problem (tile and alignment rules of its kernel).
bool gemv_w4a16_supports(const Problem &p, const qgemm_config_t &cfg);
bool gemv_w4a16_tma_supports(const Problem &p, const qgemm_config_t &cfg);
bool gemv_w4a16_h2_supports(const Problem &p, const qgemm_config_t &cfg);
bool gemv_w4a16_stream_supports(const Problem &p, const qgemm_config_t &cfg);
bool gemv_w2a8_tma_supports(const Problem &p, const qgemm_config_t &cfg);
bool gemv_int_supports(const Problem &p, const qgemm_config_t &cfg);
bool tc_supports(const Problem &p, const qgemm_config_t &cfg);
// Deepest pipeline (2..5) whose shared memory fits for this op and token tile.
int tc_max_stages(const Problem &p, int bn);
// Number of upcast-weight buffers the tensor-core kernel keeps for this ring depth (0: none).
int tc_dq_buffers(const Problem &p, int bn, int stages);

// ------------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------------

// Streaming 128/64/32-bit loads of data read exactly once (packed weights): read-only path,
// no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void *p)
{
    uint2 v;
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void *p)
{
    uint32_t v;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Cached read-only 128-bit load (activations, shared by many CTAs).
__device__ __forceinline__ uint4 ld_cached_v4(const void *p)
{
    uint4 v;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ld_cached_u16(const void *p)
{
    uint16_t v;
    asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// d = (a & b) | c  as a single LOP3 (lookup table 0xEA).
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The same with the mask and the or-pattern as immediates (compile-time constants).
template <uint32_t B, uint32_t C>
__device__ __forceinline__ uint32_t lop3_and_or_i(uint32_t a)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(B), "n"(C));
    return d;
}

// Byte permute with an immediate selector.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt_i(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "n"(SEL));
    return d;
}

// Byte permute: result byte i = byte sel_i of the 8-byte value {b:a}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ int dp4a_ss(int a, int b, int c)
{
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// a holds four UNSIGNED bytes, b four SIGNED bytes.
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Atomic adds without return (split-K epilogues).
__device__ __forceinline__ void red_add_f16x2(void *p, uint32_t v)
{
    asm volatile("red.global.add.noftz.f16x2 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 8 consecutive fp16 values (16-byte aligned)
__device__ __forceinline__ void red_add_f16x8(void *p, const uint4 &v)
{
    asm volatile("red.global.add.noftz.v4.f16x2 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void red_add_f16(void *p, uint16_t v)
{
    asm volatile("red.global.add.noftz.f16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

__device__ __forceinline__ void red_add_s32(void *p, int v)
{
    asm volatile("red.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t pack_half2_rn(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint16_t half_bits_rn(float x)
{
    __half h = __float2half_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b)
{
    __half h = *reinterpret_cast<__half *>(&b);
    return __half2float(h);
}

// Warp-level tensor-core product D = A(16x16 f16, row) . B(16x8 f16, col) + C (fp32).
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4],
                                              uint32_t b0, uint32_t b1, const float (&c)[4])
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

} // namespace qg
