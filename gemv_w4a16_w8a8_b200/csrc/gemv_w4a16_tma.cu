// W4A16 small-M streaming kernel, TMA-fed variant (group sizes that are multiples of 128).
//
// Same arithmetic plan as the register-prefetch kernel (warp-level mma.m16n8k16 with the
// weights in the 16-row slot, fp32 scale / zero per k-block), with two changes that cut the
// instruction count per weight and deepen the memory pipeline:
//   * Each warp streams its weight rows through its own ring of `STAGES` shared-memory slots
//     filled by TMA (cp.async.bulk.tensor, one elected lane), so the bytes in flight no longer
//     cost registers and no thread issues global loads for weights (hidet-org/hidet issue #364:
//     multi-stage software pipelining with a searchable stage count).
//   * The fp16 magic-number bias is not removed per weight. The LOP3 alone yields
//     x = 1024 + q (even nibbles) or 1024 + 16 q (odd nibbles); the odd-nibble activations are
//     pre-scaled by 1/16 once per k-block, so the MMA returns
//         D = sum_k a_k q_k + sum_k c_k a_k,     c_k = 1024 (even) or 64 (odd),
//     and one extra MMA per k-block against a constant operand returns, in its rows 0..7,
//     corr = sum_k c_k a_k and, in rows 8..15, sum_k a_k. Then per k-block, in fp32,
//         sum_k a_k (q_k - z) s = s * (D - corr - z * sum_k a_k).
//     Five instructions upcast eight codes; the MMA pipe absorbs the rest.
// SIMT variant for one token: the warp-level MMA issues at ~9 cycles per m16n8k16 on sm_100,
// which caps a one-token GEMV near 3 TB/s. With one token each lane instead multiplies the same
// biased codes x with its activation pairs by mixed-precision FMAs (fp16 inputs, fp32
// accumulate: every product exact), so the same five instructions plus eight FMAs handle eight
// codes; the bias sum_k c_k a_k and sum_k a_k of the lane's 32-wide K quarter are shared by all
// its rows and split over the eight lanes that hold the same quarter.
#include <mutex>

#include "sm100.cuh"

namespace qg {
namespace {

constexpr int kWarps = 4;
constexpr int kKB = 128;                 // K values per k-block (16 packed words per row)

// Activations paired like the codes the LOP3 upcast yields (natural packing: (a0,a4) (a1,a5)
// (a2,a6) (a3,a7); interleaved packing: (a0,a1) (a2,a3) (a4,a5) (a6,a7)), and the pairs that
// meet 16 q scaled by 1/16.
template <bool ILV>
__device__ __forceinline__ void act_pairs_scaled(const uint4 &v, uint32_t (&b)[4])
{
    constexpr uint32_t kInv16 = 0x2C002C00u;   // fp16 1/16 in both halves
    if constexpr (ILV) {
        b[0] = v.x;
        b[1] = hmul2_u32(v.y, kInv16);
        b[2] = v.z;
        b[3] = hmul2_u32(v.w, kInv16);
    } else {
        b[0] = prmt(v.x, v.z, 0x5410);
        b[1] = hmul2_u32(prmt(v.x, v.z, 0x7632), kInv16);
        b[2] = prmt(v.y, v.w, 0x5410);
        b[3] = hmul2_u32(prmt(v.y, v.w, 0x7632), kInv16);
    }
}

// acc + x.lo * a.lo + x.hi * a.hi, both products exact in fp32 (fp16 x fp16), two roundings
__device__ __forceinline__ float fma2_f16_f32(uint32_t x, uint32_t a, float acc)
{
    asm("{\n\t.reg .f16 xl, xh, al, ah;\n\t"
        "mov.b32 {xl, xh}, %1;\n\tmov.b32 {al, ah}, %2;\n\t"
        "fma.rn.f32.f16 %0, xl, al, %0;\n\tfma.rn.f32.f16 %0, xh, ah, %0;\n\t}"
        : "+f"(acc)
        : "r"(x), "r"(a));
    return acc;
}

template <int RB, int NT, int STAGES> struct Layout {
    static constexpr int rows = 16 * RB;
    static constexpr int slot = rows * 64;             // one stage: rows x 16 packed words
    static constexpr int tt = 8 * NT, tr = rows;
    static constexpr int ring_bytes = kWarps * STAGES * slot;
    static constexpr int bar_bytes = 8 * kWarps * STAGES;
    static constexpr int red_bytes = 4 * kWarps * tt * (tr + 1);
    static constexpr int total = ring_bytes + bar_bytes + red_bytes + 16;
};

// RB: 16-row blocks per CTA (all four warps share them and split K).  NT: 8-token tiles.
// SIMT: one token, products on the FMA pipe instead of the warp-level MMA (NT = 1, M = 1).
template <int RB, int NT, int STAGES, bool ILV, bool SIMT = false>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w4a16_tma_kernel(const __grid_constant__ CUtensorMap tm_w, const __half *__restrict__ A,
                      const __half *__restrict__ S, const __half *__restrict__ Z,
                      __half *__restrict__ C, int M, int N, int K, int gs, int kb_per_split,
                      int atomic_out, unsigned int *err, float *__restrict__ ws_part,
                      unsigned int *__restrict__ ws_count)
{
    using L = Layout<RB, NT, STAGES>;
    constexpr int kRows = L::rows, kSlot = L::slot, TT = L::tt, TR = L::tr;
    extern __shared__ __align__(128) uint8_t dsmem[];
    auto ring = reinterpret_cast<uint8_t (*)[STAGES][kSlot]>(dsmem);
    auto full = reinterpret_cast<uint64_t (*)[STAGES]>(dsmem + L::ring_bytes);
    auto red = reinterpret_cast<float (*)[TT][TR + 1]>(dsmem + L::ring_bytes + L::bar_bytes);
    int &abort_flag = *reinterpret_cast<int *>(dsmem + L::ring_bytes + L::bar_bytes + L::red_bytes);
    int &last_flag = *(&abort_flag + 1);

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lg = lane >> 2, lt = lane & 3;
    const int n0 = blockIdx.x * kRows;
    const int tok0 = blockIdx.z * TT;
    const int nkb = K / kKB;
    const int kb_begin = blockIdx.y * kb_per_split;
    const int kb_end = min(nkb, kb_begin + kb_per_split);
    if (kb_begin >= kb_end) return;
    const int G = K / gs;
    const bool zero_pt = Z != nullptr;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&full[w][s]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    __syncthreads();
    volatile int *abort_v = &abort_flag;

    // this warp's k-blocks: kb_begin + warp + kWarps * i, i < cnt
    const int first = kb_begin + warp;
    const int cnt = first < kb_end ? (kb_end - first + kWarps - 1) / kWarps : 0;
    auto issue = [&](int i) {
        const int s = i % STAGES;
        const uint32_t bar = smem_u32(&full[warp][s]);
        mbar_expect_tx(bar, kSlot);
        tma_load_2d(smem_u32(&ring[warp][s][0]), &tm_w, bar, (first + kWarps * i) * (kKB / 8),
                    n0);
    };
    if (lane == 0)
        for (int i = 0; i < min(cnt, STAGES); ++i) issue(i);
    __syncwarp();

    const __half *arow[NT];
    bool aok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        // MMA fragments: lane group lg holds token lg; SIMT: every lane holds the one token
        const int tok = SIMT ? tok0 : tok0 + 8 * t + lg;
        aok[t] = tok < M;
        arow[t] = A + (size_t)min(tok, M - 1) * K + 32 * lt;
    }
    int srow[RB][2];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
        srow[r][0] = min(n0 + 16 * r + lg, N - 1);
        srow[r][1] = min(n0 + 16 * r + lg + 8, N - 1);
    }
    float acc[RB][NT][4];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][t][i] = 0.f;

    // constant operand: rows 0..7 give sum c_k a_k, rows 8..15 give sum a_k
    const uint32_t kones[4] = {0x64006400u, 0x3C003C00u, 0x64006400u, 0x4C004C00u};
    // activations and scale / zero bits of k-block i are loaded during k-block i - 1
    uint4 av[NT][4];
    uint16_t sbits[RB][2], zbits[RB][2];
    auto prefetch = [&](int i) {
        const int k0 = (first + kWarps * i) * kKB;
        const int g = k0 / gs;
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                av[t][j] = aok[t] ? ld_cached_v4(arow[t] + k0 + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const size_t gi = (size_t)srow[r][h] * G + g;
                sbits[r][h] = ld_cached_u16(S + gi);
                zbits[r][h] = zero_pt ? ld_cached_u16(Z + gi) : (uint16_t)0;
            }
    };
    if (cnt > 0) prefetch(0);
    int consumed = 0;
    for (int i = 0; i < cnt; ++i) {
        const int s = i % STAGES;
        // take this k-block's activations and scales out of the prefetch registers
        uint32_t b[NT][4][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) act_pairs_scaled<ILV>(av[t][j], b[t][j]);
        float sc[RB][2], zr[RB][2];
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sc[r][h] = half_bits_to_float(sbits[r][h]);
                zr[r][h] = half_bits_to_float(zbits[r][h]);
            }
        if (i + 1 < cnt) prefetch(i + 1);
        if (!mbar_wait(smem_u32(&full[warp][s]), (i / STAGES) & 1, abort_v, err)) break;
        if constexpr (SIMT) {
            static_assert(NT == 1, "the SIMT inner product serves one token");
            // sum_k c_k a_k / 1024 and sum_k a_k of this lane's K quarter: the eight lanes that
            // hold the quarter (lane = 4 rq + lt) take two of its sixteen pairs each
            const int rq = lg;
            // (a, a') at weight 1 and (a / 16, a' / 16); picked with masks, not an index, so
            // that b stays in registers
            uint32_t pe = 0u, po = 0u;
            const uint32_t odd = 0u - (uint32_t)(rq & 1);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t mj = 0u - (uint32_t)((rq >> 1) == j);
                pe |= mj & ((b[0][j][2] & odd) | (b[0][j][0] & ~odd));
                po |= mj & ((b[0][j][3] & odd) | (b[0][j][1] & ~odd));
            }
            const float2 fe = __half22float2(*reinterpret_cast<const __half2 *>(&pe));
            const float2 fo = __half22float2(*reinterpret_cast<const __half2 *>(&po));
            float csum = (fe.x + fe.y) + (fo.x + fo.y);
            float asum = (fe.x + fe.y) + 16.f * (fo.x + fo.y);
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
                csum += __shfl_xor_sync(0xffffffffu, csum, m);
                asum += __shfl_xor_sync(0xffffffffu, asum, m);
            }
            const float corr = 1024.f * csum;
            const uint8_t *slot = &ring[warp][s][0];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const uint4 wa = *reinterpret_cast<const uint4 *>(slot + (16 * r + lg) * 64 + 16 * lt);
                const uint4 wb =
                    *reinterpret_cast<const uint4 *>(slot + (16 * r + lg + 8) * 64 + 16 * lt);
                const uint32_t wv[2][4] = {{wa.x, wa.y, wa.z, wa.w}, {wb.x, wb.y, wb.z, wb.w}};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float p0 = 0.f, p1 = 0.f;   // two chains
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        constexpr uint32_t kMagic = 0x64006400u, kLo = 0x000F000Fu, kHi = 0x00F000F0u;
                        const uint32_t x = wv[h][j], x8 = x >> 8;
                        p0 = fma2_f16_f32(lop3_and_or(x, kLo, kMagic), b[0][j][0], p0);
                        p1 = fma2_f16_f32(lop3_and_or(x, kHi, kMagic), b[0][j][1], p1);
                        p0 = fma2_f16_f32(lop3_and_or(x8, kLo, kMagic), b[0][j][2], p0);
                        p1 = fma2_f16_f32(lop3_and_or(x8, kHi, kMagic), b[0][j][3], p1);
                    }
                    // rows 16 r + lg (+ 8): this lane's part of s * (sum a q - z sum a)
                    acc[r][0][2 * h] += sc[r][h] * ((p0 + p1) - corr - zr[r][h] * asum);
                }
            }
        } else {
            // two independent accumulation chains per product keep the MMA pipe busy
            float cz[NT][4], cz2[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
#pragma unroll
                for (int e = 0; e < 4; ++e) cz[t][e] = cz2[t][e] = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mma_16816_f16(cz[t], kones, b[t][j][0], b[t][j][1], cz[t]);
                    mma_16816_f16(cz2[t], kones, b[t][j][2], b[t][j][3], cz2[t]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) cz[t][e] += cz2[t][e];
            }
            const uint8_t *slot = &ring[warp][s][0];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const uint4 wa = *reinterpret_cast<const uint4 *>(slot + (16 * r + lg) * 64 + 16 * lt);
                const uint4 wb =
                    *reinterpret_cast<const uint4 *>(slot + (16 * r + lg + 8) * 64 + 16 * lt);
                const uint32_t wva[4] = {wa.x, wa.y, wa.z, wa.w};
                const uint32_t wvb[4] = {wb.x, wb.y, wb.z, wb.w};
                float d[NT][4], d2[NT][4];
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[t][e] = d2[t][e] = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    constexpr uint32_t kMagic = 0x64006400u, kLo = 0x000F000Fu, kHi = 0x00F000F0u;
                    const uint32_t xa = wva[j], xb = wvb[j];
                    const uint32_t xa8 = xa >> 8, xb8 = xb >> 8;
                    const uint32_t a0[4] = {lop3_and_or(xa, kLo, kMagic), lop3_and_or(xb, kLo, kMagic),
                                            lop3_and_or(xa, kHi, kMagic), lop3_and_or(xb, kHi, kMagic)};
                    const uint32_t a1[4] = {lop3_and_or(xa8, kLo, kMagic), lop3_and_or(xb8, kLo, kMagic),
                                            lop3_and_or(xa8, kHi, kMagic), lop3_and_or(xb8, kHi, kMagic)};
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        mma_16816_f16(d[t], a0, b[t][j][0], b[t][j][1], d[t]);
                        mma_16816_f16(d2[t], a1, b[t][j][2], b[t][j][3], d2[t]);
                    }
                }
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[t][e] += d2[t][e];
                // d0 (row g, tok 2t) d1 (row g, tok 2t+1) d2 (row g+8, tok 2t) d3 (row g+8, 2t+1)
                // cz0/cz1: corr of tok 2t / 2t+1;  cz2/cz3: sum a of tok 2t / 2t+1
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    acc[r][t][0] += sc[r][0] * (d[t][0] - cz[t][0] - zr[r][0] * cz[t][2]);
                    acc[r][t][1] += sc[r][0] * (d[t][1] - cz[t][1] - zr[r][0] * cz[t][3]);
                    acc[r][t][2] += sc[r][1] * (d[t][2] - cz[t][0] - zr[r][1] * cz[t][2]);
                    acc[r][t][3] += sc[r][1] * (d[t][3] - cz[t][1] - zr[r][1] * cz[t][3]);
                }
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

    // ---- block reduction of the four warps, then store / atomic add -------------------------
    if constexpr (SIMT) {
        // acc[r][0][0] / [2]: rows 16 r + lg / 16 r + lg + 8, this lane's K quarter lt
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                float v = acc[r][0][e];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                if (lt == 0) red[warp][0][16 * r + lg + 4 * e] = v;
            }
    } else
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            red[warp][8 * t + 2 * lt][16 * r + lg] = acc[r][t][0];
            red[warp][8 * t + 2 * lt + 1][16 * r + lg] = acc[r][t][1];
            red[warp][8 * t + 2 * lt][16 * r + lg + 8] = acc[r][t][2];
            red[warp][8 * t + 2 * lt + 1][16 * r + lg + 8] = acc[r][t][3];
        }
    __syncthreads();
    if (abort_flag) return;
    if (ws_part) {
        // Deterministic split-K: park this part's fp32 tile in workspace plane blockIdx.y; the
        // last part to finish the tile sums all planes in part order and writes fp16 C.
        const int splits = gridDim.y;
        for (int e = threadIdx.x; e < TT * TR; e += kWarps * 32) {
            const int tt = e / TR, rr = e % TR;
            const int tok = tok0 + tt, row = n0 + rr;
            if (tok >= M || row >= N) continue;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += red[w][tt][rr];
            ws_part[((size_t)blockIdx.y * M + tok) * N + row] = v;
        }
        __threadfence();
        __syncthreads();
        const unsigned int tile = blockIdx.z * gridDim.x + blockIdx.x;
        if (threadIdx.x == 0)
            last_flag = atomicAdd(&ws_count[tile], 1u) == (unsigned int)(splits - 1);
        __syncthreads();
        if (!last_flag) return;
        __threadfence();
        for (int e = threadIdx.x; e < TT * TR; e += kWarps * 32) {
            const int tt = e / TR, rr = e % TR;
            const int tok = tok0 + tt, row = n0 + rr;
            if (tok >= M || row >= N) continue;
            float v = 0.f;
            for (int sp = 0; sp < splits; ++sp)
                v += __ldcg(ws_part + ((size_t)sp * M + tok) * N + row);
            C[(size_t)tok * N + row] = __float2half_rn(v);
        }
        if (threadIdx.x == 0) ws_count[tile] = 0u;   // leave the counter ready for reuse
        return;
    }
    const bool pairs = (N & 1) == 0;
    for (int e = threadIdx.x; e < TT * (TR / 2); e += kWarps * 32) {
        const int tt = e / (TR / 2);
        const int rr = 2 * (e % (TR / 2));
        const int tok = tok0 + tt;
        const int row = n0 + rr;
        if (tok >= M || row >= N) continue;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            v0 += red[w][tt][rr];
            v1 += red[w][tt][rr + 1];
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

template <int RB, int NT, int STAGES, bool ILV, bool SIMT = false>
cudaError_t launch_ilv(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream,
                       float *ws_part, unsigned int *ws_count)
{
    using L = Layout<RB, NT, STAGES>;
    auto kern = gemv_w4a16_tma_kernel<RB, NT, STAGES, ILV, SIMT>;
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
    if (!make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, p.K / 8, p.N, (uint64_t)p.K / 2,
                  kKB / 8, 16 * RB, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int nkb = p.K / kKB;
    const int kbps = (nkb + split_k - 1) / split_k;
    const int splits = (nkb + kbps - 1) / kbps;
    dim3 grid((p.N + 16 * RB - 1) / (16 * RB), splits, (p.M + 8 * NT - 1) / (8 * NT));
    kern<<<grid, kWarps * 32, L::total, stream>>>(
        tw, static_cast<const __half *>(p.A), static_cast<const __half *>(p.scales),
        p.has_zero ? static_cast<const __half *>(p.zeros) : nullptr, static_cast<__half *>(p.C),
        p.M, p.N, p.K, p.gs, kbps, (split_k > 1 && !ws_part) ? 1 : 0, err, ws_part, ws_count);
    return cudaGetLastError();
}

template <int RB, int NT, int STAGES, bool SIMT = false>
cudaError_t launch_one(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream,
                       float *ws_part, unsigned int *ws_count)
{
    return p.interleaved
               ? launch_ilv<RB, NT, STAGES, true, SIMT>(p, split_k, err, stream, ws_part, ws_count)
               : launch_ilv<RB, NT, STAGES, false, SIMT>(p, split_k, err, stream, ws_part, ws_count);
}

// one token on the FMA pipe (config bn = 1): 32, 64 or 128 rows per CTA
template <int RB>
cudaError_t launch_simt_stages(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                               cudaStream_t stream, float *wp, unsigned int *wc)
{
    switch (c.stages) {
    case 2: return launch_one<RB, 1, 2, true>(p, c.split_k, err, stream, wp, wc);
    case 3: return launch_one<RB, 1, 3, true>(p, c.split_k, err, stream, wp, wc);
    case 4: return launch_one<RB, 1, 4, true>(p, c.split_k, err, stream, wp, wc);
    case 5: return launch_one<RB, 1, 5, true>(p, c.split_k, err, stream, wp, wc);
    default: return launch_one<RB, 1, 6, true>(p, c.split_k, err, stream, wp, wc);
    }
}

template <int RB, int NT>
cudaError_t launch_stages(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                          cudaStream_t stream, float *wp, unsigned int *wc)
{
    switch (c.stages) {
    case 2: return launch_one<RB, NT, 2>(p, c.split_k, err, stream, wp, wc);
    case 3: return launch_one<RB, NT, 3>(p, c.split_k, err, stream, wp, wc);
    case 4: return launch_one<RB, NT, 4>(p, c.split_k, err, stream, wp, wc);
    case 5: return launch_one<RB, NT, 5>(p, c.split_k, err, stream, wp, wc);
    default: return launch_one<RB, NT, 6>(p, c.split_k, err, stream, wp, wc);
    }
}

template <int NT>
cudaError_t launch_rb(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream, float *wp, unsigned int *wc)
{
    if (c.rows == 16) return launch_stages<1, NT>(p, c, err, stream, wp, wc);
    if (c.rows == 32) return launch_stages<2, NT>(p, c, err, stream, wp, wc);
    return launch_stages<4, NT>(p, c, err, stream, wp, wc);
}

} // namespace

bool gemv_w4a16_tma_supports(const Problem &p, const qgemm_config_t &c)
{
    const bool stages_ok = (c.stages >= 2 && c.stages <= 6);
    const bool base = p.gs % kKB == 0 && p.K % kKB == 0 && stages_ok && c.split_k >= 1 &&
                      c.split_k <= 64;
    if (c.bn == 1)   // one token on the FMA pipe
        return base && p.M == 1 && (c.rows == 32 || c.rows == 64 || c.rows == 128);
    return base && c.bn == 0 && (c.rows == 16 || c.rows == 32 || c.rows == 64);
}

cudaError_t launch_gemv_w4a16_tma(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                                  cudaStream_t stream, float *ws_part, unsigned int *ws_count)
{
    if (c.bn == 1) {
        if (c.rows == 32) return launch_simt_stages<2>(p, c, err, stream, ws_part, ws_count);
        if (c.rows == 64) return launch_simt_stages<4>(p, c, err, stream, ws_part, ws_count);
        return launch_simt_stages<8>(p, c, err, stream, ws_part, ws_count);
    }
    if (p.M <= 8) return launch_rb<1>(p, c, err, stream, ws_part, ws_count);
    return launch_rb<2>(p, c, err, stream, ws_part, ws_count);
}

size_t gemv_w4a16_ws_tiles(const Problem &p, const qgemm_config_t &c)
{
    const int tt = p.M <= 8 ? 8 : 16;
    return (size_t)((p.N + c.rows - 1) / c.rows) * (size_t)((p.M + tt - 1) / tt);
}

} // namespace qg
