// W4A16 streaming GEMV for one to eight tokens (tiles of 1, 2 or 4) on the packed fp16 FMA pipe (group sizes that are
// multiples of 128).
//
// Why not the warp-level MMA: on sm_100 one mma.m16n8k16 occupies the legacy MMA pipe for about
// nine SM cycles and covers 256 weights, which caps a GEMV that feeds weights through it near
// 28 weights per SM cycle, below the ~45 per cycle that the measured HBM bandwidth delivers.
// Packed fp16 FMAs (HFMA2, two products per lane) have the issue budget: at one token the whole
// weight costs about two instructions (upcast, centering, product, and a share of the flush).
//
// Arithmetic, per weight row n and k-block (128 K values, inside one group g):
//   * upcast: one LOP3 puts two codes into the mantissas of fp16 1024 (x = 1024 + q for the low
//     nibble of each byte, 1024 + 16 q for the high nibble; the high nibbles need a shift by 8
//     for the second half of the word) - five instructions per eight codes;
//   * centering: q - 8 exactly, by x - 1032 (low nibbles) or x / 16 - 72 (high nibbles, one
//     HFMA2, exact because 64 + q is representable) - four instructions per eight codes;
//   * products: HFMA2 of the centred codes with activation pairs (a_k, a_k') into a half2 run
//     that covers the lane's 32 K values of the k-block (16 products per half);
//   * flush: the run's two halves go to fp32 and the group's scale and zero point are applied
//     there:  sum_k a_k (q_k - z) s = s * (sum_k a_k (q_k - 8) + (8 - z) * sum_k a_k),  with
//     sum_k a_k of the lane's 32 activations formed once per token and k-block in fp32.
// The fp16 run keeps every partial sum of 16 centred products: |a| (|q - 8| <= 8) below 512
// keeps them finite; the rounding of the run (a few units of 2^-6 at the sizes the benchmark
// uses) is scaled by s before it reaches the fp32 sum. Accumulation across k-blocks, the warps
// and split-K parts is fp32 / the output's fp16 atomics.
//
// Memory: every warp streams its own k-blocks (one in four of the CTA's K range) through a ring
// of STAGES shared-memory slots filled by TMA from one lane: the packed weights of the CTA's
// R = 8 * RPL rows (R x 64 bytes) and the NT tokens' 128 activations (NT x 256 bytes, rows
// past M read as zero) land on one mbarrier. Lane l reads 16 bytes (32 codes) of row 8 j + l / 4
// for j < RPL: one 512-byte row block per instruction, no bank conflicts. The four warps meet
// in shared memory at the end (block reduction); split-K parts meet in C through
// red.global.add.noftz.f16x2 on a zeroed C.
//
// hidet-org/hidet issue #364 ("Multi-stage software pipelining and update parallel k rule"):
// packed upcast, the multi-stage pipeline with a searchable stage count and atomic parallel-k.
#include <mutex>

#include "sm100.cuh"

namespace qg {
namespace {

constexpr int kWarps = 4;
constexpr int kKB = 128;   // K values per k-block

template <int RPL, int NT, int STAGES> struct H2Layout {
    static constexpr int rows = 8 * RPL;
    static constexpr int wbytes = rows * 64;
    static constexpr int abytes = NT * 256;
    static constexpr int slot = wbytes + abytes;     // a multiple of 128
    static constexpr int ring_bytes = kWarps * STAGES * slot;
    static constexpr int bar_bytes = 8 * kWarps * STAGES;
    static constexpr int red_bytes = 4 * kWarps * NT * rows;
    static constexpr int total = ring_bytes + bar_bytes + red_bytes + 16;
};

// x - 1032 (low nibbles: q - 8) and x / 16 - 72 (high nibbles: q - 8), both exact in fp16
__device__ __forceinline__ void centre_codes(uint32_t x, uint32_t (&w)[4])
{
    constexpr uint32_t kMagic = 0x64006400u, kLo = 0x000F000Fu, kHi = 0x00F000F0u;
    constexpr uint32_t k1032 = 0x64086408u, kInv16 = 0x2C002C00u, kNeg72 = 0xD480D480u;
    const uint32_t x8 = x >> 8;
    w[0] = hsub2_u32(lop3_and_or_i<kLo, kMagic>(x), k1032);
    w[1] = hfma2_u32(lop3_and_or_i<kHi, kMagic>(x), kInv16, kNeg72);
    w[2] = hsub2_u32(lop3_and_or_i<kLo, kMagic>(x8), k1032);
    w[3] = hfma2_u32(lop3_and_or_i<kHi, kMagic>(x8), kInv16, kNeg72);
}

// The activation pairs that meet centre_codes' output, word by word: natural packing pairs codes
// (0,4) (1,5) (2,6) (3,7) of each word; the interleaved packing pairs (0,1) (2,3) (4,5) (6,7).
template <bool ILV>
__device__ __forceinline__ void act_pairs(const uint4 &v, uint32_t (&b)[4])
{
    if constexpr (ILV) {
        b[0] = v.x;
        b[1] = v.y;
        b[2] = v.z;
        b[3] = v.w;
    } else {
        b[0] = prmt_i<0x5410>(v.x, v.z);
        b[1] = prmt_i<0x7632>(v.x, v.z);
        b[2] = prmt_i<0x5410>(v.y, v.w);
        b[3] = prmt_i<0x7632>(v.y, v.w);
    }
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

template <int RPL, int NT, int STAGES, bool ILV>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w4a16_h2_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                     const __half *__restrict__ S, const __half *__restrict__ Z,
                     __half *__restrict__ C, int M, int N, int K, int gs, int kb_per_split,
                     int atomic_out, unsigned int *err)
{
    using L = H2Layout<RPL, NT, STAGES>;
    constexpr int R = L::rows;
    extern __shared__ __align__(128) uint8_t dsmem[];
    auto ring = reinterpret_cast<uint8_t (*)[STAGES][L::slot]>(dsmem);
    auto full = reinterpret_cast<uint64_t (*)[STAGES]>(dsmem + L::ring_bytes);
    auto red = reinterpret_cast<float (*)[NT][R]>(dsmem + L::ring_bytes + L::bar_bytes);
    int &abort_flag =
        *reinterpret_cast<int *>(dsmem + L::ring_bytes + L::bar_bytes + L::red_bytes);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lg = lane >> 2, lt = lane & 3;
    const int n0 = blockIdx.x * R;
    const int tok0 = blockIdx.z * NT;
    const int nkb = K / kKB;
    const int kb_begin = blockIdx.y * kb_per_split;
    const int kb_end = min(nkb, kb_begin + kb_per_split);
    if (kb_begin >= kb_end) return;
    const int G = K / gs;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&full[w][s]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    __syncthreads();
    volatile int *abort_v = &abort_flag;

    // this warp's k-blocks: first + kWarps * i, i < cnt
    const int first = kb_begin + warp;
    const int cnt = first < kb_end ? (kb_end - first + kWarps - 1) / kWarps : 0;
    auto issue = [&](int i) {
        const int s = i % STAGES;
        const uint32_t bar = smem_u32(&full[warp][s]);
        const int kb = first + kWarps * i;
        mbar_expect_tx(bar, L::slot);
        tma_load_2d(smem_u32(&ring[warp][s][0]), &tm_w, bar, kb * (kKB / 8), n0);
        tma_load_2d(smem_u32(&ring[warp][s][L::wbytes]), &tm_a, bar, kb * kKB, tok0);
    };
    if (lane == 0)
        for (int i = 0; i < min(cnt, STAGES); ++i) issue(i);
    __syncwarp();

    // this lane's rows n0 + 8 j + lg (clamped for the scale / zero reads; the tail is masked)
    int srow[RPL];
#pragma unroll
    for (int j = 0; j < RPL; ++j) srow[j] = min(n0 + 8 * j + lg, N - 1);
    float acc[RPL][NT];
#pragma unroll
    for (int j = 0; j < RPL; ++j)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[j][t] = 0.f;

    // scale / zero bits of k-block i are loaded during k-block i - 1
    uint16_t sbits[RPL], zbits[RPL];
    auto prefetch_sz = [&](int i) {
        const int g = (first + kWarps * i) * kKB / gs;
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            const size_t gi = (size_t)srow[j] * G + g;
            sbits[j] = ld_cached_u16(S + gi);
            zbits[j] = Z ? ld_cached_u16(Z + gi) : (uint16_t)0;
        }
    };
    if (cnt > 0) prefetch_sz(0);
    int consumed = 0;
    for (int i = 0; i < cnt; ++i) {
        const int s = i % STAGES;
        float sc[RPL], cz[RPL];
#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            sc[j] = half_bits_to_float(sbits[j]);
            cz[j] = 8.f - half_bits_to_float(zbits[j]);
        }
        if (i + 1 < cnt) prefetch_sz(i + 1);
        const uint32_t fbar = smem_u32(&full[warp][s]);
        if (!(mbar_try_wait(fbar, (i / STAGES) & 1) ||
              mbar_wait(fbar, (i / STAGES) & 1, abort_v, err)))
            break;
        const uint8_t *slot = &ring[warp][s][0];

        // activations of this lane's 32 K values, paired like the codes; their sum in fp32
        uint32_t ap[NT][4][4];
        float asum[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            uint32_t q4[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 av =
                    *reinterpret_cast<const uint4 *>(slot + L::wbytes + 256 * t + 64 * lt + 16 * v);
                act_pairs<ILV>(av, ap[t][v]);
                // pairwise sums of the word's eight activations (two fp16 additions deep)
                q4[v] = hadd2_u32(hadd2_u32(av.x, av.y), hadd2_u32(av.z, av.w));
            }
            const float2 f0 = half2_bits_to_float2(q4[0]), f1 = half2_bits_to_float2(q4[1]);
            const float2 f2 = half2_bits_to_float2(q4[2]), f3 = half2_bits_to_float2(q4[3]);
            asum[t] = ((f0.x + f0.y) + (f1.x + f1.y)) + ((f2.x + f2.y) + (f3.x + f3.y));
        }

#pragma unroll
        for (int j = 0; j < RPL; ++j) {
            const uint4 wv = *reinterpret_cast<const uint4 *>(slot + (8 * j + lg) * 64 + 16 * lt);
            const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
            uint32_t run[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) run[t] = 0u;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
                centre_codes(words[v], w);
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) run[t] = hfma2_u32(w[e], ap[t][v][e], run[t]);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                // the run's two halves meet in fp16 (sums of 16 centred products each), then the
                // group's scale and zero point apply in fp32
                const uint32_t both = hadd2_u32(run[t], prmt_i<0x1032>(run[t], run[t]));
                const float f = __half2float(*reinterpret_cast<const __half *>(&both));
                acc[j][t] = fmaf(sc[j], fmaf(cz[j], asum[t], f), acc[j][t]);
            }
        }
        consumed = i + 1;
        // slot s is free again: refill it with k-block i + STAGES
        __syncwarp();
        if (lane == 0 && i + STAGES < cnt) {
            fence_proxy_async_smem();
            issue(i + STAGES);
        }
    }
    // copies still in flight (only after a bounded wait gave up) must land before exit
    if (lane == 0) {
        int dummy = 0;
        for (int i = consumed; i < min(cnt, consumed + STAGES); ++i)
            mbar_wait(smem_u32(&full[warp][i % STAGES]), (i / STAGES) & 1, &dummy, nullptr);
    }

    // ---- the four K quarters of each row (lanes lt), then the four warps ---------------------
#pragma unroll
    for (int j = 0; j < RPL; ++j)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            float v = acc[j][t];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            if (lt == 0) red[warp][t][8 * j + lg] = v;
        }
    __syncthreads();
    if (abort_flag) return;
    const bool pairs = (N & 1) == 0;
    for (int e = threadIdx.x; e < NT * (R / 2); e += kWarps * 32) {
        const int t = e / (R / 2);
        const int rr = 2 * (e % (R / 2));
        const int tok = tok0 + t, row = n0 + rr;
        if (tok >= M || row >= N) continue;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            v0 += red[w][t][rr];
            v1 += red[w][t][rr + 1];
        }
        __half *dst = C + (size_t)tok * N + row;
        if (pairs) {
            const uint32_t hv = pack_half2_rn(v0, v1);
            if (atomic_out) red_add_f16x2(dst, hv);
            else *reinterpret_cast<uint32_t *>(dst) = hv;
        } else {
            if (atomic_out) red_add_f16(dst, half_bits_rn(v0));
            else dst[0] = __float2half_rn(v0);
            if (row + 1 < N) {
                if (atomic_out) red_add_f16(dst + 1, half_bits_rn(v1));
                else dst[1] = __float2half_rn(v1);
            }
        }
    }
}

template <int RPL, int NT, int STAGES, bool ILV>
cudaError_t launch_h2(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream)
{
    using L = H2Layout<RPL, NT, STAGES>;
    auto kern = gemv_w4a16_h2_kernel<RPL, NT, STAGES, ILV>;
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
    CUtensorMap tw, ta;
    if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, p.K / 8, p.N, (uint64_t)p.K / 2,
                  kKB / 8, L::rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.A, p.K, p.M, (uint64_t)p.K * 2, kKB, NT,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int nkb = p.K / kKB;
    const int kbps = (nkb + split_k - 1) / split_k;
    const int splits = (nkb + kbps - 1) / kbps;
    dim3 grid((p.N + L::rows - 1) / L::rows, splits, (p.M + NT - 1) / NT);
    kern<<<grid, kWarps * 32, L::total, stream>>>(
        tw, ta, static_cast<const __half *>(p.scales),
        p.has_zero ? static_cast<const __half *>(p.zeros) : nullptr, static_cast<__half *>(p.C),
        p.M, p.N, p.K, p.gs, kbps, split_k > 1 ? 1 : 0, err);
    return cudaGetLastError();
}

template <int RPL, int NT, int STAGES>
cudaError_t launch_layout(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream)
{
    return p.interleaved ? launch_h2<RPL, NT, STAGES, true>(p, split_k, err, stream)
                         : launch_h2<RPL, NT, STAGES, false>(p, split_k, err, stream);
}

template <int RPL, int NT>
cudaError_t launch_stages(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                          cudaStream_t stream)
{
    switch (c.stages) {
    case 2: return launch_layout<RPL, NT, 2>(p, c.split_k, err, stream);
    case 3: return launch_layout<RPL, NT, 3>(p, c.split_k, err, stream);
    case 4: return launch_layout<RPL, NT, 4>(p, c.split_k, err, stream);
    case 5: return launch_layout<RPL, NT, 5>(p, c.split_k, err, stream);
    default: return launch_layout<RPL, NT, 6>(p, c.split_k, err, stream);
    }
}

template <int NT>
cudaError_t launch_rows(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                        cudaStream_t stream)
{
    if (c.rows == 32) return launch_stages<4, NT>(p, c, err, stream);
    return launch_stages<8, NT>(p, c, err, stream);
}

} // namespace

// Token tile of the half2 kernel for M tokens: 1, 2 or 4 (larger M runs several tiles).
int gemv_w4a16_h2_tokens(int M) { return M <= 1 ? 1 : (M == 2 ? 2 : 4); }

bool gemv_w4a16_h2_supports(const Problem &p, const qgemm_config_t &c)
{
    return c.path == QG_PATH_GEMV && c.bn == 2 && (c.rows == 32 || c.rows == 64) &&
           c.stages >= 2 && c.stages <= 6 && c.split_k >= 1 && c.split_k <= 64 && p.M <= 8 &&
           p.gs % kKB == 0 && p.K % kKB == 0;
}

cudaError_t launch_gemv_w4a16_h2(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                                 cudaStream_t stream)
{
    switch (gemv_w4a16_h2_tokens(p.M)) {
    case 1: return launch_rows<1>(p, c, err, stream);
    case 2: return launch_rows<2>(p, c, err, stream);
    default: return launch_rows<4>(p, c, err, stream);
    }
}

} // namespace qg
