// Weight packing kernels: uint8 int4 codes -> 8 per uint32, int8 int2 values -> 16 per uint32.
// Element k of a row lands at bits 4*(k%8) (int4) or 2*(k%16) (int2) of word k/8 (k/16); the
// interleaved layouts permute the elements inside each word (see the kernels).
// Each thread turns 16 output bytes' worth of input into one 128-bit store.
#include <algorithm>

#include "common.cuh"

namespace qg {
namespace {

// four codes (bytes of x, low nibbles) -> 16 bits, code i at bits 4i
__device__ __forceinline__ uint32_t nibbles4(uint32_t x)
{
    x &= 0x0F0F0F0Fu;
    x = (x | (x >> 4)) & 0x00FF00FFu;
    return (x | (x >> 8)) & 0x0000FFFFu;
}

// four 2-bit fields (bytes of x, low 2 bits) -> 8 bits, field i at bits 2i
__device__ __forceinline__ uint32_t fields4(uint32_t x)
{
    x &= 0x03030303u;
    x = (x | (x >> 6)) & 0x000F000Fu;
    return (x | (x >> 12)) & 0x000000FFu;
}

__global__ void pack_int4_kernel(const uint8_t *__restrict__ codes, uint32_t *__restrict__ packed,
                                 size_t units)
{
    // unit u: 32 codes (two 16-byte loads) -> 4 words (one 16-byte store)
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units;
         u += (size_t)gridDim.x * blockDim.x) {
        const uint4 a = ld_stream_v4(codes + 32 * u);
        const uint4 b = ld_stream_v4(codes + 32 * u + 16);
        uint4 o;
        o.x = nibbles4(a.x) | (nibbles4(a.y) << 16);
        o.y = nibbles4(a.z) | (nibbles4(a.w) << 16);
        o.z = nibbles4(b.x) | (nibbles4(b.y) << 16);
        o.w = nibbles4(b.z) | (nibbles4(b.w) << 16);
        reinterpret_cast<uint4 *>(packed)[u] = o;
    }
}

// interleaved layout: the even codes of a word fill its low 16 bits, the odd codes its high 16
__global__ void pack_int4_interleaved_kernel(const uint8_t *__restrict__ codes,
                                             uint32_t *__restrict__ packed, size_t units)
{
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units;
         u += (size_t)gridDim.x * blockDim.x) {
        const uint4 a = ld_stream_v4(codes + 32 * u);
        const uint4 b = ld_stream_v4(codes + 32 * u + 16);
        const uint32_t lo[4] = {a.x, a.z, b.x, b.z}, hi[4] = {a.y, a.w, b.y, b.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = nibbles4(prmt(lo[q], hi[q], 0x6420)) | (nibbles4(prmt(lo[q], hi[q], 0x7531)) << 16);
        reinterpret_cast<uint4 *>(packed)[u] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void pack_int2_kernel(const int8_t *__restrict__ vals, uint32_t *__restrict__ packed,
                                 size_t units)
{
    // unit u: 64 values (four 16-byte loads) -> 4 words (one 16-byte store)
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units;
         u += (size_t)gridDim.x * blockDim.x) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 a = ld_stream_v4(vals + 64 * u + 16 * q);
            w[q] = fields4(a.x) | (fields4(a.y) << 8) | (fields4(a.z) << 16) |
                   (fields4(a.w) << 24);
        }
        reinterpret_cast<uint4 *>(packed)[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// interleaved int2 layout: fields 0..15 of a word hold values 0,4,1,5,2,6,3,7, 8,12,9,13,10,14,11,15
__global__ void pack_int2_interleaved_kernel(const int8_t *__restrict__ vals,
                                             uint32_t *__restrict__ packed, size_t units)
{
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units;
         u += (size_t)gridDim.x * blockDim.x) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 a = ld_stream_v4(vals + 64 * u + 16 * q);
            w[q] = fields4(prmt(a.x, a.y, 0x5140)) | (fields4(prmt(a.x, a.y, 0x7362)) << 8) |
                   (fields4(prmt(a.z, a.w, 0x5140)) << 16) |
                   (fields4(prmt(a.z, a.w, 0x7362)) << 24);
        }
        reinterpret_cast<uint4 *>(packed)[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

int grid_for(size_t units)
{
    const size_t want = (units + 255) / 256;
    return (int)(want < 148 * 16 ? (want ? want : 1) : 148 * 16);
}

// Round-to-nearest int4 quantisation of fp16 weights (the header states the rule). One warp per
// span of max(group_size, 256) K values of one row; lane l holds K values 8l .. 8l+7 of each
// 256-wide chunk, i.e. exactly packed word l of the chunk. Groups narrower than 256 are reduced
// over their gs / 8 lanes with butterfly shuffles, wider ones over the whole warp and chunk
// loop. Every value that decides a code is computed in binary32 with correctly rounded
// division and rintf (half to even).
__global__ void rtn_int4_kernel(const __half *__restrict__ W, uint32_t *__restrict__ Wq,
                                __half *__restrict__ S, __half *__restrict__ Z, int K, int gs,
                                long long tasks)
{
    const int lane = threadIdx.x & 31;
    const long long first = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    const long long stride = (gridDim.x * (long long)blockDim.x) >> 5;
    // narrow groups: spans of 256 (the last one of a row may be shorter; it still holds whole
    // groups, so a lane past the row's end only shares a group with lanes past it too)
    const int span = gs < 256 ? 256 : gs;
    const int spans = (K + span - 1) / span;
    const int G = K / gs;
    const int lanes = gs < 256 ? gs / 8 : 32;   // lanes that share a group (a power of two)
    for (long long t = first; t < tasks; t += stride) {
        const long long n = t / spans;
        const int sp = (int)(t - n * spans);
        const bool active = sp * span + 8 * lane < K;
        const __half *w = W + (size_t)n * K + (size_t)sp * span;
        float lo = 0.0f, hi = 0.0f;
        uint4 keep = make_uint4(0u, 0u, 0u, 0u);   // the values of a single-chunk span
        for (int c = 0; c < span; c += 256) {
            const uint4 v = active ? ld_stream_v4(w + c + 8 * lane) : make_uint4(0u, 0u, 0u, 0u);
            keep = v;
            const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hv[i]));
                lo = fminf(lo, fminf(f.x, f.y));
                hi = fmaxf(hi, fmaxf(f.x, f.y));
            }
        }
        for (int off = 1; off < lanes; off <<= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        const float range = hi - lo;
        const float s32 = range > 0.0f ? __fdiv_rn(range, 15.0f) : 1.0f;
        __half s16 = __float2half_rn(s32);
        if ((__half_as_ushort(s16) & 0x7FFFu) == 0) s16 = __ushort_as_half((unsigned short)1);
        const float sf = __half2float(s16);
        const float z = fminf(fmaxf(rintf(0.0f - __fdiv_rn(lo, sf)), 0.0f), 15.0f);
        const int g = gs < 256 ? (sp * 256 + 8 * lane) / gs : sp;
        if (!active) continue;   // (no shuffles follow)
        if ((lane & (lanes - 1)) == 0) {
            S[(size_t)n * G + g] = s16;
            Z[(size_t)n * G + g] = __float2half_rn(z);
        }
        for (int c = 0; c < span; c += 256) {
            const uint4 v = span == 256 ? keep : ld_stream_v4(w + c + 8 * lane);
            const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hv[i]));
                const float q0 = fminf(fmaxf(rintf(__fdiv_rn(f.x, sf)) + z, 0.0f), 15.0f);
                const float q1 = fminf(fmaxf(rintf(__fdiv_rn(f.y, sf)) + z, 0.0f), 15.0f);
                word |= ((uint32_t)q0 << (8 * i)) | ((uint32_t)q1 << (8 * i + 4));
            }
            Wq[((size_t)n * K + (size_t)sp * span + c) / 8 + lane] = word;
        }
    }
}

} // namespace

cudaError_t launch_pack_int4(const uint8_t *codes, uint32_t *packed, int N, int K,
                             cudaStream_t stream)
{
    const size_t units = (size_t)N * K / 32;   // K % 32 == 0 keeps units inside rows
    pack_int4_kernel<<<grid_for(units), 256, 0, stream>>>(codes, packed, units);
    return cudaGetLastError();
}

cudaError_t launch_pack_int4_interleaved(const uint8_t *codes, uint32_t *packed, int N, int K,
                                         cudaStream_t stream)
{
    const size_t units = (size_t)N * K / 32;
    pack_int4_interleaved_kernel<<<grid_for(units), 256, 0, stream>>>(codes, packed, units);
    return cudaGetLastError();
}

cudaError_t launch_pack_int2(const int8_t *vals, uint32_t *packed, int N, int K,
                             cudaStream_t stream)
{
    const size_t units = (size_t)N * K / 64;
    pack_int2_kernel<<<grid_for(units), 256, 0, stream>>>(vals, packed, units);
    return cudaGetLastError();
}

cudaError_t launch_pack_int2_interleaved(const int8_t *vals, uint32_t *packed, int N, int K,
                                         cudaStream_t stream)
{
    const size_t units = (size_t)N * K / 64;
    pack_int2_interleaved_kernel<<<grid_for(units), 256, 0, stream>>>(vals, packed, units);
    return cudaGetLastError();
}

cudaError_t launch_rtn_int4(const __half *W, uint32_t *Wq, __half *S, __half *Z, int N, int K,
                            int gs, cudaStream_t stream)
{
    const int span = gs < 256 ? 256 : gs;
    const long long tasks = (long long)N * ((K + span - 1) / span);
    const long long blocks = std::min<long long>((tasks + 7) / 8, 148LL * 32);
    rtn_int4_kernel<<<(unsigned)std::max(1LL, blocks), 256, 0, stream>>>(W, Wq, S, Z, K, gs, tasks);
    return cudaGetLastError();
}

} // namespace qg
