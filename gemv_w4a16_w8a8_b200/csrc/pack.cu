// Weight packing kernels: uint8 int4 codes -> 8 per uint32, int8 int2 values -> 16 per uint32.
// Element k of a row lands at bits 4*(k%8) (int4) or 2*(k%16) (int2) of word k/8 (k/16).
// Each thread turns 16 output bytes' worth of input into one 128-bit store.
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

int grid_for(size_t units)
{
    const size_t want = (units + 255) / 256;
    return (int)(want < 148 * 16 ? (want ? want : 1) : 148 * 16);
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

} // namespace qg
