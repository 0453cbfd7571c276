// W8A8 / W2A8 small-M streaming kernels (int8 activations, int32 results).
//
// Each warp owns R weight rows and walks K in 16-byte chunks of the packed weight row (16 int8
// values, or 64 int2 values), one chunk per lane per step, so a warp step reads 512 contiguous
// bytes of every row with 128-bit loads. Products are formed with dp4a into int32, the lanes
// are combined with a butterfly of warp shuffles, and split-K parts meet in C through
// red.global.add.s32 (exact: integer addition is associative). Results are bit-exact.
//
// int2 upcast (two's complement fields u in 0..3 meaning u - 4*(u>>1)): with u' = u ^ 2 the
// value is u' - 2 and u' is an unsigned 2-bit number. XOR-ing the word with 0xAAAAAAAA forms
// all sixteen u' at once; (w' >> 2j) & 0x03030303 puts fields j, j+4, j+8, j+12 into the four
// bytes of one register, which dp4a multiplies (unsigned x signed) against the activations
// gathered the same way with two rounds of PRMT (one round for the interleaved layout). The
// -2 * sum(a) correction is one more dp4a per activation register, shared by all rows of the
// warp.
#include "common.cuh"

namespace qg {
namespace {

constexpr int kWarps = 4;
constexpr int kUnroll = 2;     // chunks per lane loaded before any is consumed

__device__ __forceinline__ int warp_sum(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// bytes (a_j, a_{j+4}, a_{j+8}, a_{j+12}) for j = 0..3 from natural-order a0..a15
__device__ __forceinline__ void gather_stride4(const uint32_t r0, const uint32_t r1,
                                               const uint32_t r2, const uint32_t r3,
                                               uint32_t (&p)[4])
{
    const uint32_t t0 = prmt(r0, r1, 0x5140);   // r0.b0 r1.b0 r0.b1 r1.b1
    const uint32_t t1 = prmt(r0, r1, 0x7362);   // r0.b2 r1.b2 r0.b3 r1.b3
    const uint32_t t2 = prmt(r2, r3, 0x5140);
    const uint32_t t3 = prmt(r2, r3, 0x7362);
    p[0] = prmt(t0, t2, 0x5410);
    p[1] = prmt(t0, t2, 0x7632);
    p[2] = prmt(t1, t3, 0x5410);
    p[3] = prmt(t1, t3, 0x7632);
}

// The same for the interleaved int2 layout, whose fields j, j+4, j+8, j+12 hold values
// (0,2,8,10), (4,6,12,14), (1,3,9,11), (5,7,13,15) for j = 0..3: one round of PRMT.
__device__ __forceinline__ void gather_interleaved(const uint32_t r0, const uint32_t r1,
                                                   const uint32_t r2, const uint32_t r3,
                                                   uint32_t (&p)[4])
{
    p[0] = prmt(r0, r2, 0x6420);
    p[1] = prmt(r1, r3, 0x6420);
    p[2] = prmt(r0, r2, 0x7531);
    p[3] = prmt(r1, r3, 0x7531);
}

// R rows per warp, MT tokens per CTA. INT2 selects the packed 2-bit weight format, ILV its
// interleaved layout.
template <int R, int MT, bool INT2, bool ILV = false>
__global__ void __launch_bounds__(kWarps * 32)
gemv_int_kernel(const int8_t *__restrict__ A, const uint8_t *__restrict__ W,
                int32_t *__restrict__ C, int M, int N, int K, int chunks_per_split,
                int atomic_out, const float *__restrict__ mult)
{
    constexpr int KC = INT2 ? 64 : 16;           // K values per 16-byte weight chunk
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int n0 = (blockIdx.x * kWarps + warp) * R;
    const int m0 = blockIdx.z * MT;
    const int nchunks = K / KC;
    const int c_begin = blockIdx.y * chunks_per_split;
    const int c_end = min(nchunks, c_begin + chunks_per_split);
    const size_t row_bytes = INT2 ? (size_t)K / 4 : (size_t)K;
    if (n0 >= N || c_begin >= c_end) return;

    const uint8_t *wrow[R];
    bool wok[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        wok[r] = n0 + r < N;
        wrow[r] = W + (size_t)min(n0 + r, N - 1) * row_bytes;
    }
    const int8_t *arow[MT];
    bool aok[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        aok[t] = m0 + t < M;
        arow[t] = A + (size_t)min(m0 + t, M - 1) * K;
    }

    int acc[R][MT];
    int asum[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        asum[t] = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r][t] = 0;
    }

    for (int c0 = c_begin + lane; c0 < c_end; c0 += 32 * kUnroll) {
        uint4 wv[kUnroll][R];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int c = c0 + 32 * u;
#pragma unroll
            for (int r = 0; r < R; ++r)
                wv[u][r] = (c < c_end && wok[r]) ? ld_stream_v4(wrow[r] + (size_t)c * 16)
                                                 : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int c = c0 + 32 * u;
            if (c >= c_end) break;
            if constexpr (!INT2) {
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    const uint4 a = aok[t] ? ld_cached_v4(arow[t] + (size_t)c * 16)
                                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        int s = acc[r][t];
                        s = dp4a_ss((int)wv[u][r].x, (int)a.x, s);
                        s = dp4a_ss((int)wv[u][r].y, (int)a.y, s);
                        s = dp4a_ss((int)wv[u][r].z, (int)a.z, s);
                        s = dp4a_ss((int)wv[u][r].w, (int)a.w, s);
                        acc[r][t] = s;
                    }
                }
            } else {
                // 64 activations per token: natural order -> the stride-4 byte order of the
                // fields, per 16-value word
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    uint32_t ap[4][4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 a = aok[t] ? ld_cached_v4(arow[t] + (size_t)c * 64 + 16 * q)
                                               : make_uint4(0u, 0u, 0u, 0u);
                        if constexpr (ILV) gather_interleaved(a.x, a.y, a.z, a.w, ap[q]);
                        else gather_stride4(a.x, a.y, a.z, a.w, ap[q]);
                        int s = asum[t];
                        s = dp4a_ss(0x01010101, (int)a.x, s);
                        s = dp4a_ss(0x01010101, (int)a.y, s);
                        s = dp4a_ss(0x01010101, (int)a.z, s);
                        s = dp4a_ss(0x01010101, (int)a.w, s);
                        asum[t] = s;
                    }
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint32_t words[4] = {wv[u][r].x, wv[u][r].y, wv[u][r].z, wv[u][r].w};
                        int s = acc[r][t];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t wf = words[q] ^ 0xAAAAAAAAu;
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                s = dp4a_us((wf >> (2 * j)) & 0x03030303u, (int)ap[q][j], s);
                        }
                        acc[r][t] = s;
                    }
                }
            }
        }
    }

#pragma unroll
    for (int t = 0; t < MT; ++t) {
        const int corr = INT2 ? 2 * warp_sum(asum[t]) : 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int v = warp_sum(acc[r][t]) - corr;
            if (lane == 0 && wok[r] && aok[t]) {
                const size_t idx = (size_t)(m0 + t) * N + n0 + r;
                if (mult) reinterpret_cast<int8_t *>(C)[idx] = requant_i8(v, mult[n0 + r]);
                else if (atomic_out) red_add_s32(C + idx, v);
                else C[idx] = v;
            }
        }
    }
}

template <int R, int MT, bool INT2>
void launch_one(const Problem &p, int split_k, cudaStream_t stream)
{
    constexpr int KC = INT2 ? 64 : 16;
    const int nchunks = p.K / KC;
    const int cps = (nchunks + split_k - 1) / split_k;
    const int splits = (nchunks + cps - 1) / cps;
    dim3 grid((p.N + kWarps * R - 1) / (kWarps * R), splits, (p.M + MT - 1) / MT);
    auto kern = (INT2 && p.interleaved) ? gemv_int_kernel<R, MT, INT2, true>
                                        : gemv_int_kernel<R, MT, INT2, false>;
    kern<<<grid, kWarps * 32, 0, stream>>>(
        static_cast<const int8_t *>(p.A), static_cast<const uint8_t *>(p.W),
        static_cast<int32_t *>(p.C), p.M, p.N, p.K, cps, split_k > 1 ? 1 : 0, p.mult);
}

template <int R, bool INT2>
void launch_mt(const Problem &p, int split_k, cudaStream_t stream)
{
    if (p.M == 1) launch_one<R, 1, INT2>(p, split_k, stream);
    else if (p.M == 2) launch_one<R, 2, INT2>(p, split_k, stream);
    else launch_one<R, 4, INT2>(p, split_k, stream);
}

template <bool INT2>
void launch_r(const Problem &p, int rows, int split_k, cudaStream_t stream)
{
    switch (rows) {
    case 1: launch_mt<1, INT2>(p, split_k, stream); break;
    case 2: launch_mt<2, INT2>(p, split_k, stream); break;
    case 8: launch_mt<8, INT2>(p, split_k, stream); break;
    default: launch_mt<4, INT2>(p, split_k, stream); break;
    }
}

} // namespace

bool gemv_int_supports(const Problem &p, const qgemm_config_t &cfg)
{
    const int kc = p.op == QG_OP_W2A8 ? 64 : 16;
    return p.K % kc == 0 && cfg.stages == 0 && (cfg.rows == 1 || cfg.rows == 2 || cfg.rows == 4 || cfg.rows == 8) &&
           cfg.split_k >= 1 && cfg.split_k <= 64;
}

cudaError_t launch_gemv_int(const Problem &p, const qgemm_config_t &cfg, cudaStream_t stream)
{
    if (p.op == QG_OP_W2A8) launch_r<true>(p, cfg.rows, cfg.split_k, stream);
    else launch_r<false>(p, cfg.rows, cfg.split_k, stream);
    return cudaGetLastError();
}

} // namespace qg
