// W4A16 small-M streaming kernel: C[M,N] = A[M,K] . ((q - z) * s)^T for M up to 16 per CTA.
//
// The weights are the only large operand, so the kernel is built to stream them from HBM once
// with 128-bit loads, keep several k-blocks of them in flight per warp, and spend as few
// instructions per weight as possible (hidet-org/hidet issue #364, "Multi-stage software
// pipelining and update parallel k rule": vectorised ("packed") upcasting and parallel-k).
//
// Per weight the SIMT cost of an fp32-accurate fused multiply-add on B200 would exceed the
// issue budget at HBM speed as soon as M >= 2, so the multiply-accumulate runs on the
// warp-level tensor-core instruction mma.m16n8k16 (weights in the 16-row A slot, up to 8 tokens
// in the B slot), and the CUDA cores only upcast:
//   * one LOP3 with the fp16 exponent pattern of 1024.0 turns a nibble pair into the exact
//     fp16 pair (1024 + q_i, 1024 + q_{i+4}) (or (1024 + 16 q, ...) for the odd nibbles), one
//     HSUB2 / HFMA2 removes the bias exactly; 9 instructions give the 8 codes of a word;
//   * the order inside a word is (0,4),(1,5),(2,6),(3,7); K may be permuted freely as long as
//     A is permuted the same way, so the activations are paired the same way with PRMT.
// Scale and zero are applied per k-block (a k-block never straddles a group):
//     sum_k a_k (q_k - z) s = s * (sum_k a_k q_k - z * sum_k a_k)
// where sum_k a_k comes from one extra MMA against an all-ones A operand.
// Split-K parts are reduced inside the CTA through shared memory (block reduction) and across
// CTAs with red.global.add.noftz.f16x2 into a C that the host zeroed.
#include "common.cuh"

namespace qg {
namespace {

constexpr int kWarps = 4;
constexpr int kPrefetch = 3;   // k-blocks of weights in flight per warp

template <int WPT>
__device__ __forceinline__ void load_words(uint32_t (&w)[WPT], const uint32_t *p)
{
    if constexpr (WPT == 4) {
        uint4 v = ld_stream_v4(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (WPT == 2) {
        uint2 v = ld_stream_v2(p);
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = ld_stream_u32(p);
    }
}

// Exact fp16 pairs of the eight codes of one word: (q0,q4) (q1,q5) (q2,q6) (q3,q7) for the
// natural packing, (q0,q1) (q2,q3) (q4,q5) (q6,q7) for the interleaved one.
__device__ __forceinline__ void upcast_word(uint32_t w, uint32_t (&h)[4])
{
    constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 | 1024.0
    constexpr uint32_t kLo = 0x000F000Fu;
    constexpr uint32_t kHi = 0x00F000F0u;
    constexpr uint32_t kInv16 = 0x2C002C00u;  // fp16 0.0625 | 0.0625
    constexpr uint32_t kNeg64 = 0xD400D400u;  // fp16 -64 | -64
    const uint32_t w8 = w >> 8;
    h[0] = hsub2_u32(lop3_and_or(w, kLo, kMagic), kMagic);
    h[1] = hfma2_u32(lop3_and_or(w, kHi, kMagic), kInv16, kNeg64);
    h[2] = hsub2_u32(lop3_and_or(w8, kLo, kMagic), kMagic);
    h[3] = hfma2_u32(lop3_and_or(w8, kHi, kMagic), kInv16, kNeg64);
}

// Eight activations (h0..h7) paired to match upcast_word: (h0,h4) (h1,h5) (h2,h6) (h3,h7) for
// the natural packing; for the interleaved packing upcast_word yields (q0,q1) (q2,q3) (q4,q5)
// (q6,q7), so the activations stay in natural pairs and need no permutation.
template <bool ILV>
__device__ __forceinline__ void act_pairs(const uint4 &v, uint32_t (&b)[4])
{
    if constexpr (ILV) {
        b[0] = v.x; b[1] = v.y; b[2] = v.z; b[3] = v.w;
    } else {
        b[0] = prmt(v.x, v.z, 0x5410);
        b[1] = prmt(v.x, v.z, 0x7632);
        b[2] = prmt(v.y, v.w, 0x5410);
        b[3] = prmt(v.y, v.w, 0x7632);
    }
}

// WPT: packed words per thread per row per k-block (k-block = 32*WPT values of K).
// RB:  16-row blocks per warp.  NT: 8-token tiles per CTA.
template <int WPT, int RB, int NT, bool ILV>
__global__ void __launch_bounds__(kWarps * 32)
gemv_w4a16_kernel(const __half *__restrict__ A, const uint32_t *__restrict__ Wq,
                  const __half *__restrict__ S, const __half *__restrict__ Z,
                  __half *__restrict__ C, int M, int N, int K, int gs, int kb_per_split,
                  int atomic_out)
{
    constexpr int KB = 32 * WPT;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lg = lane >> 2;   // row (A operand) / token (B operand) inside the fragment
    const int lt = lane & 3;
    const int n0 = blockIdx.x * 16 * RB;
    const int tok0 = blockIdx.z * 8 * NT;
    const int nkb = K / KB;
    const int kb_begin = blockIdx.y * kb_per_split;
    const int kb_end = min(nkb, kb_begin + kb_per_split);
    const int G = K / gs;
    const size_t wpr = (size_t)K / 8;   // packed words per row
    const bool zero_pt = Z != nullptr;

    if (kb_begin >= kb_end) return;     // empty split: C was zeroed by the host

    const uint32_t *wrow[RB][2];
    bool wok[RB][2];
    int wr[RB][2];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = n0 + 16 * r + lg + 8 * h;
            wok[r][h] = row < N;
            wr[r][h] = min(row, N - 1);
            wrow[r][h] = Wq + (size_t)wr[r][h] * wpr + lt * WPT;
        }
    const __half *arow[NT];
    bool aok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int tok = tok0 + 8 * t + lg;
        aok[t] = tok < M;
        arow[t] = A + (size_t)min(tok, M - 1) * K + 8 * lt * WPT;
    }

    float acc[RB][NT][4];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[r][t][i] = 0.f;

    uint32_t wbuf[kPrefetch][RB][2][WPT];

    auto load_kb = [&](uint32_t (&dst)[RB][2][WPT], int kb) {
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (wok[r][h]) {
                    load_words<WPT>(dst[r][h], wrow[r][h] + (size_t)kb * (KB / 8));
                } else {
#pragma unroll
                    for (int j = 0; j < WPT; ++j) dst[r][h][j] = 0u;
                }
            }
    };

    auto compute_kb = [&](const uint32_t (&wv)[RB][2][WPT], int kb) {
        // activations for this k-block, re-paired
        uint32_t b[NT][WPT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int j = 0; j < WPT; ++j) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (aok[t]) v = ld_cached_v4(arow[t] + (size_t)kb * KB + 8 * j);
                act_pairs<ILV>(v, b[t][j]);
            }
        const int g = (kb * KB) / gs;
        float s[RB][2], z[RB][2];
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const size_t gi = (size_t)wr[r][h] * G + g;
                s[r][h] = wok[r][h] ? half_bits_to_float(ld_cached_u16(S + gi)) : 0.f;
                z[r][h] = zero_pt ? half_bits_to_float(ld_cached_u16(Z + gi)) : 0.f;
            }
        // sum of the activations of this k-block per token (needed only with zero points)
        float asum[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i) asum[t][i] = 0.f;
        if (zero_pt) {
            const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int j = 0; j < WPT; ++j) {
                    mma_16816_f16(asum[t], ones, b[t][j][0], b[t][j][1], asum[t]);
                    mma_16816_f16(asum[t], ones, b[t][j][2], b[t][j][3], asum[t]);
                }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            float d[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) d[t][i] = 0.f;
#pragma unroll
            for (int j = 0; j < WPT; ++j) {
                uint32_t qa[4], qb[4];
                upcast_word(wv[r][0][j], qa);
                upcast_word(wv[r][1][j], qb);
                const uint32_t a0[4] = {qa[0], qb[0], qa[1], qb[1]};
                const uint32_t a1[4] = {qa[2], qb[2], qa[3], qb[3]};
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    mma_16816_f16(d[t], a0, b[t][j][0], b[t][j][1], d[t]);
                    mma_16816_f16(d[t], a1, b[t][j][2], b[t][j][3], d[t]);
                }
            }
            // fragment: d0 (row g, tok 2t) d1 (row g, tok 2t+1) d2 (row g+8, tok 2t) d3 (...)
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                acc[r][t][0] += s[r][0] * (d[t][0] - z[r][0] * asum[t][0]);
                acc[r][t][1] += s[r][0] * (d[t][1] - z[r][0] * asum[t][1]);
                acc[r][t][2] += s[r][1] * (d[t][2] - z[r][1] * asum[t][0]);
                acc[r][t][3] += s[r][1] * (d[t][3] - z[r][1] * asum[t][1]);
            }
        }
    };

    // software pipeline over this warp's k-blocks: kb_begin + warp, + kWarps, ...
    const int first = kb_begin + warp;
#pragma unroll
    for (int p = 0; p < kPrefetch; ++p) {
        const int kb = first + p * kWarps;
        if (kb < kb_end) load_kb(wbuf[p], kb);
    }
    for (int kb = first; kb < kb_end; kb += kPrefetch * kWarps) {
#pragma unroll
        for (int p = 0; p < kPrefetch; ++p) {
            const int kbp = kb + p * kWarps;
            if (kbp < kb_end) {
                compute_kb(wbuf[p], kbp);
                const int kbn = kbp + kPrefetch * kWarps;
                if (kbn < kb_end) load_kb(wbuf[p], kbn);
            }
        }
    }

    // ---- block reduction of the four warps' partial sums, then store / atomic add ----------
    constexpr int TT = 8 * NT;      // tokens in the CTA tile
    constexpr int TR = 16 * RB;     // rows in the CTA tile
    __shared__ float red[kWarps][TT][TR + 1];
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
        if (pairs) {   // row even and N even: dst is 4-byte aligned and row + 1 < N
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

template <int WPT, int RB, int NT, bool ILV>
void launch_ilv(const Problem &p, int split_k, cudaStream_t stream)
{
    constexpr int KB = 32 * WPT;
    const int nkb = p.K / KB;
    const int kbps = (nkb + split_k - 1) / split_k;
    const int splits = (nkb + kbps - 1) / kbps;   // drop trailing empty splits
    dim3 grid((p.N + 16 * RB - 1) / (16 * RB), splits, (p.M + 8 * NT - 1) / (8 * NT));
    gemv_w4a16_kernel<WPT, RB, NT, ILV><<<grid, kWarps * 32, 0, stream>>>(
        static_cast<const __half *>(p.A), static_cast<const uint32_t *>(p.W),
        static_cast<const __half *>(p.scales),
        p.has_zero ? static_cast<const __half *>(p.zeros) : nullptr, static_cast<__half *>(p.C),
        p.M, p.N, p.K, p.gs, kbps, split_k > 1 ? 1 : 0);
}

template <int WPT, int RB, int NT>
void launch_one(const Problem &p, int split_k, cudaStream_t stream)
{
    if (p.interleaved) launch_ilv<WPT, RB, NT, true>(p, split_k, stream);
    else launch_ilv<WPT, RB, NT, false>(p, split_k, stream);
}

template <int WPT, int NT>
void launch_rb(const Problem &p, int rows, int split_k, cudaStream_t stream)
{
    if (rows == 16) launch_one<WPT, 1, NT>(p, split_k, stream);
    else if (rows == 64) launch_one<WPT, 4, NT>(p, split_k, stream);
    else launch_one<WPT, 2, NT>(p, split_k, stream);
}

template <int WPT>
void launch_nt(const Problem &p, int rows, int split_k, cudaStream_t stream)
{
    if (p.M <= 8) launch_rb<WPT, 1>(p, rows, split_k, stream);
    else launch_rb<WPT, 2>(p, rows, split_k, stream);
}

} // namespace

bool gemv_w4a16_supports(const Problem &p, const qgemm_config_t &cfg)
{
    return p.K % 32 == 0 && p.gs % 32 == 0 && p.K % p.gs == 0 && cfg.stages == 0 && cfg.bn == 0 &&
           (cfg.rows == 16 || cfg.rows == 32 || cfg.rows == 64) && cfg.split_k >= 1 &&
           cfg.split_k <= 64;
}

cudaError_t launch_gemv_w4a16(const Problem &p, const qgemm_config_t &cfg, cudaStream_t stream)
{
    // widest k-block that stays inside one quantisation group
    if (p.gs % 128 == 0) launch_nt<4>(p, cfg.rows, cfg.split_k, stream);
    else if (p.gs % 64 == 0) launch_nt<2>(p, cfg.rows, cfg.split_k, stream);
    else launch_nt<1>(p, cfg.rows, cfg.split_k, stream);
    return cudaGetLastError();
}

} // namespace qg
