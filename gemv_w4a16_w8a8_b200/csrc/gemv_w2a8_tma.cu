// W2A8 small-M streaming kernel, TMA-fed: int8 activations x two's-complement int2 weights.
//
// Each warp streams its k-blocks (256 values of K = 16 packed words per weight row) through a
// private ring of shared-memory slots filled by TMA, and multiplies on the warp-level tensor-core
// instruction mma.m16n8k32 with unsigned 8-bit weights and signed 8-bit activations, int32
// accumulation across the whole K range (exact: no per-block scaling exists for this format).
// Upcast: XOR with 0xAAAAAAAA turns every field u into u' = u ^ 2 (the value is u' - 2, with u'
// an unsigned 0..3), and (w' >> 2j) & 0x03030303 (j = 0..3) places fields j, j+4, j+8, j+12 in
// the bytes of one register - 9 instructions for 16 weights. The activations are regathered
// once per k-block into the same byte order with two rounds of PRMT (one round for the
// interleaved int2 layout, whose fields hold a different fixed permutation of K), and one extra MMA against
// an all-ones operand yields sum_k a_k, so that C = sum_k a_k u'_k - 2 sum_k a_k.
#include <mutex>

#include "sm100.cuh"

namespace qg {
namespace {

constexpr int kWarps = 4;
constexpr int kKB = 256;                 // K values per k-block (16 packed words per row)

__device__ __forceinline__ void mma_16832_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bytes (a_j, a_{j+4}, a_{j+8}, a_{j+12}) for j = 0..3 from natural-order a0..a15
__device__ __forceinline__ void gather4(const uint4 &v, uint32_t (&p)[4])
{
    const uint32_t t0 = prmt(v.x, v.y, 0x5140), t1 = prmt(v.x, v.y, 0x7362);
    const uint32_t t2 = prmt(v.z, v.w, 0x5140), t3 = prmt(v.z, v.w, 0x7362);
    p[0] = prmt(t0, t2, 0x5410);
    p[1] = prmt(t0, t2, 0x7632);
    p[2] = prmt(t1, t3, 0x5410);
    p[3] = prmt(t1, t3, 0x7632);
}

// the same for the interleaved layout, whose fields j, j+4, j+8, j+12 hold values (0,2,8,10),
// (4,6,12,14), (1,3,9,11), (5,7,13,15) for j = 0..3
__device__ __forceinline__ void gather4_interleaved(const uint4 &v, uint32_t (&p)[4])
{
    p[0] = prmt(v.x, v.z, 0x6420);
    p[1] = prmt(v.y, v.w, 0x6420);
    p[2] = prmt(v.x, v.z, 0x7531);
    p[3] = prmt(v.y, v.w, 0x7531);
}

template <int RB, int NT, int STAGES> struct Layout {
    static constexpr int rows = 16 * RB;
    static constexpr int slot = rows * 64;
    static constexpr int tt = 8 * NT, tr = rows;
    static constexpr int ring_bytes = kWarps * STAGES * slot;
    static constexpr int bar_bytes = 8 * kWarps * STAGES;
    static constexpr int red_bytes = 4 * kWarps * tt * (tr + 1);
    static constexpr int total = ring_bytes + bar_bytes + red_bytes + 16;
};

template <int RB, int NT, int STAGES, bool ILV>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w2a8_tma_kernel(const __grid_constant__ CUtensorMap tm_w, const int8_t *__restrict__ A,
                     int32_t *__restrict__ C, int M, int N, int K, int kb_per_split,
                     int atomic_out, unsigned int *err)
{
    using L = Layout<RB, NT, STAGES>;
    constexpr int kRows = L::rows, kSlot = L::slot, TT = L::tt, TR = L::tr;
    extern __shared__ __align__(128) uint8_t dsmem[];
    auto ring = reinterpret_cast<uint8_t (*)[STAGES][kSlot]>(dsmem);
    auto full = reinterpret_cast<uint64_t (*)[STAGES]>(dsmem + L::ring_bytes);
    auto red = reinterpret_cast<int (*)[TT][TR + 1]>(dsmem + L::ring_bytes + L::bar_bytes);
    int &abort_flag = *reinterpret_cast<int *>(dsmem + L::ring_bytes + L::bar_bytes + L::red_bytes);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lg = lane >> 2, lt = lane & 3;
    const int n0 = blockIdx.x * kRows;
    const int tok0 = blockIdx.z * TT;
    const int nkb = K / kKB;
    const int kb_begin = blockIdx.y * kb_per_split;
    const int kb_end = min(nkb, kb_begin + kb_per_split);
    if (kb_begin >= kb_end) return;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&full[w][s]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    __syncthreads();
    volatile int *abort_v = &abort_flag;

    const int first = kb_begin + warp;
    const int cnt = first < kb_end ? (kb_end - first + kWarps - 1) / kWarps : 0;
    auto issue = [&](int i) {
        const int s = i % STAGES;
        const uint32_t bar = smem_u32(&full[warp][s]);
        mbar_expect_tx(bar, kSlot);
        tma_load_2d(smem_u32(&ring[warp][s][0]), &tm_w, bar, (first + kWarps * i) * (kKB / 16),
                    n0);
    };
    if (lane == 0)
        for (int i = 0; i < min(cnt, STAGES); ++i) issue(i);
    __syncwarp();

    const int8_t *arow[NT];
    bool aok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int tok = tok0 + 8 * t + lg;
        aok[t] = tok < M;
        arow[t] = A + (size_t)min(tok, M - 1) * K + 64 * lt;   // thread lt: words 4lt..4lt+3
    }
    // two independent accumulation chains per product keep the MMA pipe busy
    int acc[RB][NT][4], acc2[RB][NT][4];
    int asum[NT][4], asum2[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) asum[t][e] = asum2[t][e] = 0;
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][t][e] = acc2[r][t][e] = 0;
    }
    const uint32_t kOnes[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};

    int consumed = 0;
    for (int i = 0; i < cnt; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(smem_u32(&full[warp][s]), (i / STAGES) & 1, abort_v, err)) break;
        const int k0 = (first + kWarps * i) * kKB;
        // activations of this k-block: 4 words x 16 values per thread, regathered
        uint32_t b[NT][4][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (aok[t]) v = ld_cached_v4(arow[t] + k0 + 16 * q);
                if constexpr (ILV) gather4_interleaved(v, b[t][q]);
                else gather4(v, b[t][q]);
                mma_16832_u8s8(asum[t], kOnes, b[t][q][0], b[t][q][1]);
                mma_16832_u8s8(asum2[t], kOnes, b[t][q][2], b[t][q][3]);
            }
        const uint8_t *slot = &ring[warp][s][0];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const uint4 wa = *reinterpret_cast<const uint4 *>(slot + (16 * r + lg) * 64 + 16 * lt);
            const uint4 wb =
                *reinterpret_cast<const uint4 *>(slot + (16 * r + lg + 8) * 64 + 16 * lt);
            const uint32_t wva[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wvb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t fa = wva[q] ^ 0xAAAAAAAAu, fb = wvb[q] ^ 0xAAAAAAAAu;
                const uint32_t a0[4] = {fa & 0x03030303u, fb & 0x03030303u,
                                        (fa >> 2) & 0x03030303u, (fb >> 2) & 0x03030303u};
                const uint32_t a1[4] = {(fa >> 4) & 0x03030303u, (fb >> 4) & 0x03030303u,
                                        (fa >> 6) & 0x03030303u, (fb >> 6) & 0x03030303u};
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    mma_16832_u8s8(acc[r][t], a0, b[t][q][0], b[t][q][1]);
                    mma_16832_u8s8(acc2[r][t], a1, b[t][q][2], b[t][q][3]);
                }
            }
        }
        consumed = i + 1;
        __syncwarp();
        if (lane == 0 && i + STAGES < cnt) {
            fence_proxy_async_smem();
            issue(i + STAGES);
        }
    }
    if (lane == 0) {
        int dummy = 0;
        for (int i = consumed; i < min(cnt, consumed + STAGES); ++i)
            mbar_wait(smem_u32(&full[warp][i % STAGES]), (i / STAGES) & 1, &dummy, nullptr);
    }

    // C = sum a u' - 2 sum a; fragment: e0 (row g, tok 2t) e1 (row g, 2t+1) e2/e3 (row g+8)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            asum[t][e] += asum2[t][e];
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r][t][e] += acc2[r][t][e];
        }
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            red[warp][8 * t + 2 * lt][16 * r + lg] = acc[r][t][0] - 2 * asum[t][0];
            red[warp][8 * t + 2 * lt + 1][16 * r + lg] = acc[r][t][1] - 2 * asum[t][1];
            red[warp][8 * t + 2 * lt][16 * r + lg + 8] = acc[r][t][2] - 2 * asum[t][2];
            red[warp][8 * t + 2 * lt + 1][16 * r + lg + 8] = acc[r][t][3] - 2 * asum[t][3];
        }
    __syncthreads();
    if (abort_flag) return;
    for (int e = threadIdx.x; e < TT * TR; e += kWarps * 32) {
        const int tt = e / TR, rr = e % TR;
        const int tok = tok0 + tt, row = n0 + rr;
        if (tok >= M || row >= N) continue;
        int v = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][tt][rr];
        int32_t *dst = C + (size_t)tok * N + row;
        if (atomic_out) red_add_s32(dst, v);
        else *dst = v;
    }
}

template <int RB, int NT, int STAGES, bool ILV>
cudaError_t launch_layout(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream)
{
    using L = Layout<RB, NT, STAGES>;
    auto kern = gemv_w2a8_tma_kernel<RB, NT, STAGES, ILV>;
    static std::mutex mu;
    static bool opted_in[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!opted_in[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 L::total);
            if (e != cudaSuccess) return e;
            opted_in[dev] = true;
        }
    }
    CUtensorMap tw;
    if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, p.K / 16, p.N, (uint64_t)p.K / 4,
                  kKB / 16, 16 * RB, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int nkb = p.K / kKB;
    const int kbps = (nkb + split_k - 1) / split_k;
    const int splits = (nkb + kbps - 1) / kbps;
    dim3 grid((p.N + 16 * RB - 1) / (16 * RB), splits, (p.M + 8 * NT - 1) / (8 * NT));
    kern<<<grid, kWarps * 32, L::total, stream>>>(tw, static_cast<const int8_t *>(p.A),
                                                  static_cast<int32_t *>(p.C), p.M, p.N, p.K,
                                                  kbps, split_k > 1 ? 1 : 0, err);
    return cudaGetLastError();
}

template <int RB, int NT, int STAGES>
cudaError_t launch_one(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream)
{
    return p.interleaved ? launch_layout<RB, NT, STAGES, true>(p, split_k, err, stream)
                         : launch_layout<RB, NT, STAGES, false>(p, split_k, err, stream);
}

template <int RB, int NT>
cudaError_t launch_stages(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                          cudaStream_t stream)
{
    switch (c.stages) {
    case 2: return launch_one<RB, NT, 2>(p, c.split_k, err, stream);
    case 3: return launch_one<RB, NT, 3>(p, c.split_k, err, stream);
    case 4: return launch_one<RB, NT, 4>(p, c.split_k, err, stream);
    case 5: return launch_one<RB, NT, 5>(p, c.split_k, err, stream);
    default: return launch_one<RB, NT, 6>(p, c.split_k, err, stream);
    }
}

template <int NT>
cudaError_t launch_rb(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream)
{
    if (c.rows == 16) return launch_stages<1, NT>(p, c, err, stream);
    if (c.rows == 32) return launch_stages<2, NT>(p, c, err, stream);
    return launch_stages<4, NT>(p, c, err, stream);
}

} // namespace

bool gemv_w2a8_tma_supports(const Problem &p, const qgemm_config_t &c)
{
    return p.op == QG_OP_W2A8 && p.K % kKB == 0 && (c.rows == 16 || c.rows == 32 || c.rows == 64) &&
           (c.stages >= 2 && c.stages <= 6) && c.split_k >= 1 &&
           c.split_k <= 64;
}

cudaError_t launch_gemv_w2a8_tma(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                                 cudaStream_t stream)
{
    if (p.M <= 8) return launch_rb<1>(p, c, err, stream);
    return launch_rb<2>(p, c, err, stream);
}

} // namespace qg
