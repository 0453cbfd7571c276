// tcgen05 tensor-core GEMM family (dense fp16, W8A8, W4A16, W2A8): tcgen05.mma with operands in
// shared memory and the accumulator in TMEM, fed by TMA, one persistent CTA of 512 threads per
// SM walking work units (weight tile, token tile, K part).
//
// Two tile orientations, because an MMA from shared memory at M = 128 occupies the tensor pipe
// ~98 cycles for any N up to 128 and reaches its full rate only at N = 256 (measured):
//   weight-major   D[128 weight rows, BN tokens] = W_tile . A_tile^T, BN in {16..256}; the
//                  large-M tile (BN = 256) upcasts each weight once per 256 tokens, and the
//                  512-token tile of the packed formats feeds each upcast slab to two N = 256
//                  MMAs (two accumulators filling TMEM), once per 512 tokens;
//   token-major    D[128 tokens, 256 weight rows] = A_tile . W_tile^T (W4A16): tokens are the A
//                  operand (rows past M read as zero), 256 upcast weight rows the B operand, so
//                  every MMA runs at N = 256 for 1..128 tokens.
//
// Roles (warp-specialised):
//   warp 4      TMA producer of the activation ring (and the weight slab for fp16 / int8
//               weights): STAGES 128-byte-wide K slabs under SWIZZLE_128B, mbarrier transaction
//               counts (multi-stage software pipelining with a tunable stage count, as the
//               num_stages search in hidet-org/hidet issue #364);
//   warp 6      TMA producer of the packed-weight ring (4-slab copies: 128 contiguous bytes of
//               each weight row);
//   warp 5      TMEM allocation and the MMA issue, one slab at a time, each slab's buffers
//               committed back to their producers as soon as its MMAs complete;
//   warps 8-15  upcast of packed weights into the K-major SWIZZLE_128B layout the MMA reads
//               (LOP3 magic-number upcast, PRMT re-ordering, HFMA2 with the group's scale and
//               zero), handed over per slab or per copy;
//   warps 0-3   epilogue: tcgen05.ld of the (double-buffered) accumulator, conversion, stores or
//               red.global.add for split-K and stream-K (parallel-k through atomics, hidet issue
//               #364); weight-major fp16 results leave as 16-byte rows after a shuffle transpose.
// Work units: whole tiles, K parts of them (split-K), or equal shares of the flattened (tile, K)
// work per persistent CTA (stream-K).
// Every wait is bounded (%globaltimer); a wait that runs out raises the device error word, makes
// the other roles stop, lets in-flight copies land, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace qg {
namespace {

enum Mode { kDense = 0, kW8A8 = 1, kW4A16 = 2, kW2A8 = 3, kW4A16I = 4, kW2A8I = 5 };   // I: interleaved

constexpr bool is_w4(int m) { return m == kW4A16 || m == kW4A16I; }
constexpr bool is_w2(int m) { return m == kW2A8 || m == kW2A8I; }

constexpr int kThreads = 512;
constexpr int kRowsW = 128;            // weight rows per tile (MMA M)
// Token-major variant (TOKA) for few tokens: the tokens are the MMA's A operand (M = 128; rows
// past the last token read as zero) and 256 upcast weight rows its B operand (N = 256). An MMA
// from shared memory costs the same ~100 cycles for any N up to 128 and reaches the full rate
// only at N = 256, so few tokens in N waste most of the tensor core; in M they do not.
constexpr int kRowsT = 256;            // weight rows per tile of the token-major variant
constexpr int kTokT = 128;             // tokens per tile of the token-major variant
template <bool TOKA> constexpr int wrows() { return TOKA ? kRowsT : kRowsW; }
constexpr int kSlabBytes = 128;        // bytes of K per stage and row (64 fp16 / 128 int8)
constexpr int kGroupT = 8;             // token tiles per raster group

// Shared-memory matrix descriptor: K-major, SWIZZLE_128B, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
    d |= (uint64_t)1 << 16;                          // leading byte offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8 rows
    d |= (uint64_t)1 << 46;                          // descriptor version
    d |= (uint64_t)2 << 61;                          // swizzle: 128B
    return d;
}

template <int MODE>
__device__ __forceinline__ void mma_issue(uint32_t dtm, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate)
{
    if constexpr (MODE == kDense || is_w4(MODE)) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtm),
                     "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtm),
                     "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                     : "memory");
    }
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// ---- CTA pairs (cta_group::2): one MMA spans the tensor cores of two SMs of a cluster --------
// The leader (rank 0) issues every MMA; A's 256 rows are the two CTAs' 128-row weight slabs and
// B's N rows the two CTAs' halves of the token tile, each read from its own CTA's shared memory
// at the same offset; each CTA's TMEM holds the accumulator rows of its own weight rows.

template <int MODE>
__device__ __forceinline__ void mma_issue_pair(uint32_t dtm, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t accumulate)
{
    if constexpr (MODE == kDense || is_w4(MODE)) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtm),
                     "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtm),
                     "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                     : "memory");
    }
}

// arrive on the barrier at the same offset in both CTAs of the pair once the MMAs finish
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::"
                 "cluster.b64 [%0], %1;" ::"r"(bar), "h"((uint16_t)3)
                 : "memory");
}

// arrive on this CTA's own barrier once the MMAs finish
__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// address of the same shared-memory location in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// arrival (release at cluster scope) on a barrier given by its shared::cluster address
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// every thread of both CTAs
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// 2-D TMA load into this CTA's shared memory that completes its bytes on a barrier of either
// CTA of the pair (given by its shared::cluster address); no multicast
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar_cluster, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx"
                 "::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                   "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Instruction descriptor: dense, K-major A and B, M = MR (128, or 256 for a CTA pair), N = BN.
//   fp16 x fp16 -> fp32: D format 1, A/B format 0.   int8 x int8 -> int32: D 2, A/B 1 (signed).
template <int MODE, int BN, int MR = kRowsW>
__host__ __device__ constexpr uint32_t instr_desc()
{
    constexpr bool i8 = (MODE == kW8A8 || is_w2(MODE));
    return (i8 ? 2u : 1u) << 4 | (i8 ? 1u : 0u) << 7 | (i8 ? 1u : 0u) << 10 |
           (uint32_t)(BN >> 3) << 17 | (uint32_t)(MR >> 4) << 24;
}

template <int MODE> struct Traits {
    static constexpr bool packed = (is_w4(MODE) || is_w2(MODE));
    static constexpr int w_tma_bytes = packed ? kRowsW * 32 : kRowsW * kSlabBytes;
    static constexpr int w_mma_bytes = packed ? kRowsW * kSlabBytes : 0;   // dequant target
    static constexpr int k_per_slab = (MODE == kDense || is_w4(MODE)) ? 64 : 128;
    static constexpr int c_bytes = (MODE == kDense || is_w4(MODE)) ? 2 : 4;
};

// Shared memory.
//   dense / int8 weights: one ring of STAGES stages, each a weight slab and an activation slab
//     loaded by TMA (SWIZZLE_128B) and read by the MMA.
//   packed weights: three rings, so that no latency of one step sits in the cycle of another:
//     STAGES activation slabs (TMA -> MMA), sp packed-weight copies of PG slabs each (TMA ->
//     upcast, so the upcast can run far ahead; see packed_stages) and DQ upcast weight slabs
//     (upcast -> MMA; see dq_buffers).
constexpr int kMaxSmem = 227 * 1024;

// Packed weights move PG slabs per copy: PG = 4 reads 128 contiguous bytes of each weight row
// (HBM serves long row runs far better than 32-byte ones); PG = 1 when K is not a multiple of
// four slabs.
//
// Upcast weight buffers go from the dequantisation warps to the MMA either one slab at a time
// (token tiles of 128 and more: an MMA slab is long enough to hide a hand-over, and the MMA must
// not wait for a whole copy) or one packed copy at a time (smaller tiles: there the hand-overs
// themselves are the cost, and one proxy fence and one arrival per copy are paid instead of PG).
constexpr bool per_slab_handoff(int bn) { return bn >= 128; }
// one word per dequantisation thread (see the release of a packed copy)
constexpr int kSinkBytes = 256 * 4;
// the fewest upcast buffers a plan may have, and how many it should keep before the packed ring
// gives up copies for them
constexpr int min_dq(int pg, int bn) { return (pg < 2 || per_slab_handoff(bn)) ? 2 : pg; }
constexpr int want_dq(int pg, int bn) { return per_slab_handoff(bn) ? 3 : min_dq(pg, bn); }

// Activation rows of one stage held by a CTA: the token tile; half of it for a CTA pair; 256 for
// the 512-token tile, whose slabs arrive as two 256-token stages (one per accumulator).
constexpr int act_rows(int bn, bool pair) { return pair ? bn / 2 : (bn > 256 ? 256 : bn); }

// ar: activation rows of a stage held by this CTA (the MMA's N, or half of it for a CTA pair)
constexpr int smem_total(bool packed, int ar, int stages, int dq, int pg, int sp, int wr = kRowsW)
{
    return packed ? 1024 + stages * ar * kSlabBytes + sp * wr * 32 * pg + dq * wr * kSlabBytes +
                        kSinkBytes + 8 * (2 * stages + 2 * sp + 2 * dq + 5) + 16
                  : 1024 + stages * (kRowsW * kSlabBytes + ar * kSlabBytes) + 8 * (2 * stages + 5) +
                        16;
}

// Packed-weight copies in flight: 12 single slabs, or 6 / 4 grouped copies; for token tiles of
// 128 and more, fewer when a deep activation ring would otherwise leave less than want_dq upcast
// buffers (one grouped copy holds 4 slabs, so 2-3 copies already run far ahead of the MMA).
constexpr int packed_stages(int pg, int bn, int stages, int wr = kRowsW, int ar = 0)
{
    if (pg == 1) return 12;
    if (bn <= 64) return 6;
    const int a = ar ? ar : bn;
    int sp = 4;
    while (sp > 2 && smem_total(true, a, stages, want_dq(pg, bn), pg, sp, wr) > kMaxSmem) --sp;
    return sp;
}

// Upcast-weight buffers: as many as fit, up to 8. Each buffer makes a round trip (upcast, fence,
// arrive, MMA, commit, release) whose latency bounds the throughput when the token tile is small,
// so small tiles take the most. A plan below min_dq is reported as not fitting (smem_bytes).
constexpr int dq_buffers(bool packed, int bn, int stages, int pg, int wr = kRowsW, int ar = 0)
{
    if (!packed) return 0;
    const int a = ar ? ar : bn;
    const int sp = packed_stages(pg, bn, stages, wr, a);
    int d = 8;
    while (d > min_dq(pg, bn) && smem_total(true, a, stages, d, pg, sp, wr) > kMaxSmem) --d;
    return d;
}

// BN: tokens per tile (the MMA's N, or its M in the token-major variant); WR weight rows of this
// CTA. PAIR: a CTA pair shares each MMA (cta_group::2), and each CTA holds half of the tile's
// tokens (AR rows of every activation stage).
template <int MODE, int BN, int STAGES, int PG, bool TOKA = false, bool PAIR = false> struct Smem {
    static constexpr bool packed = Traits<MODE>::packed;
    static constexpr int WR = wrows<TOKA>();
    static constexpr int AR = act_rows(BN, PAIR);
    static constexpr int a_bytes = AR * kSlabBytes;
    static constexpr int w_bytes = kRowsW * kSlabBytes;          // dense / int8 weight slab
    static constexpr int pw_bytes = WR * 32 * PG;                // packed weight copy (PG slabs)
    static constexpr int sp = packed ? packed_stages(PG, BN, STAGES, WR, AR) : 0;
    static constexpr int dq = dq_buffers(packed, BN, STAGES, PG, WR, AR);
    static constexpr int dq_bytes = WR * kSlabBytes;
    // byte offsets from the 1024-aligned base
    static constexpr int ring_bytes = packed ? STAGES * a_bytes : STAGES * (w_bytes + a_bytes);
    static constexpr int pw_off = ring_bytes;
    static constexpr int dq_off = pw_off + sp * pw_bytes;
    static constexpr int sink_off = dq_off + dq * dq_bytes;
    static constexpr int bar_off = sink_off + (packed ? kSinkBytes : 0);
    static constexpr int nbars = 2 * STAGES + 2 * sp + 2 * dq + 5;
    static constexpr int total = smem_total(packed, AR, STAGES, dq, PG, sp, WR);
};

// two accumulator buffers of BN fp32 / int32 columns (the allocation is a power of two >= 32)
template <int BN> constexpr uint32_t tmem_cols() { return 2 * BN < 32 ? 32u : (uint32_t)(2 * BN); }

// Upcast half a slab of packed int4 (p = words 4h..4h+3 of weight row r: 32 values of K, one
// quantisation group) into fp16 (q - z) * s = fma(q, s, fp16(-z * s)), written in the
// SWIZZLE_128B K-major layout the MMA reads.
template <bool ILV>
__device__ __forceinline__ void dequant_w4(const uint4 &p, uint8_t *dst, int r, int h,
                                           uint32_t sc, uint32_t nz)
{
    constexpr uint32_t kMagic = 0x64006400u, kLo = 0x000F000Fu, kHi = 0x00F000F0u;
    constexpr uint32_t kInv16 = 0x2C002C00u, kNeg64 = 0xD400D400u;
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    uint8_t *row = dst + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = words[j], w8 = w >> 8;
        // natural packing: (q0,q4) (q1,q5) (q2,q6) (q3,q7); interleaved: (q0,q1) .. (q6,q7)
        const uint32_t h0 = hsub2_u32(lop3_and_or_i<kLo, kMagic>(w), kMagic);
        const uint32_t h1 = hfma2_u32(lop3_and_or_i<kHi, kMagic>(w), kInv16, kNeg64);
        const uint32_t h2 = hsub2_u32(lop3_and_or_i<kLo, kMagic>(w8), kMagic);
        const uint32_t h3 = hfma2_u32(lop3_and_or_i<kHi, kMagic>(w8), kInv16, kNeg64);
        uint4 o;
        if constexpr (ILV) {
            o.x = hfma2_u32(h0, sc, nz);
            o.y = hfma2_u32(h1, sc, nz);
            o.z = hfma2_u32(h2, sc, nz);
            o.w = hfma2_u32(h3, sc, nz);
        } else {
            o.x = hfma2_u32(prmt_i<0x5410>(h0, h1), sc, nz);   // (q0, q1)
            o.y = hfma2_u32(prmt_i<0x5410>(h2, h3), sc, nz);   // (q2, q3)
            o.z = hfma2_u32(prmt_i<0x7632>(h0, h1), sc, nz);   // (q4, q5)
            o.w = hfma2_u32(prmt_i<0x7632>(h2, h3), sc, nz);   // (q6, q7)
        }
        *reinterpret_cast<uint4 *>(row + (((4 * h + j) ^ (r & 7)) << 4)) = o;
    }
}

// Upcast half a slab of packed int2 (p = words 4h..4h+3 of weight row r: 64 values) into int8.
// Byte-table lookup: PRMT with both sources holding the int8 values of the four 2-bit codes
// (0, 1, -2, -1 -> 0x00, 0x01, 0xFE, 0xFF) turns the low three bits of each selector nibble into
// a byte (bit 2 picks the second, identical copy of the table), so (w >> s) & 0x7777 for
// s = 0, 2, 16, 18 gives the values of fields (0,2,4,6), (1,3,5,7), (8,10,12,14), (9,11,13,15).
// In the interleaved layout those are values 0-3, 4-7, 8-11, 12-15 in K order (11 instructions
// a word); the natural layout needs one more byte transpose of register pairs (15).
template <bool ILV>
__device__ __forceinline__ void dequant_w2(const uint4 &p, uint8_t *dst, int r, int h)
{
    constexpr uint32_t kTable = 0xFFFE0100u, kSel = 0x7777u;
    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
    uint8_t *row = dst + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = words[j];
        const uint32_t d0 = prmt(kTable, kTable, w & kSel);
        const uint32_t d1 = prmt(kTable, kTable, (w >> 2) & kSel);
        const uint32_t d2 = prmt(kTable, kTable, (w >> 16) & kSel);
        const uint32_t d3 = prmt(kTable, kTable, (w >> 18) & kSel);
        uint4 o;
        if constexpr (ILV) {
            o = make_uint4(d0, d1, d2, d3);
        } else {
            o.x = prmt_i<0x5140>(d0, d1);   // values 0, 1, 2, 3
            o.y = prmt_i<0x7362>(d0, d1);   // 4 .. 7
            o.z = prmt_i<0x5140>(d2, d3);   // 8 .. 11
            o.w = prmt_i<0x7362>(d2, d3);   // 12 .. 15
        }
        *reinterpret_cast<uint4 *>(row + (((4 * h + j) ^ (r & 7)) << 4)) = o;
    }
}

__device__ __forceinline__ uint32_t half2_bcast(float x)
{
    const uint16_t b = half_bits_rn(x);
    return (uint32_t)b | ((uint32_t)b << 16);
}

// Weight-major fp16 epilogue: 16 tokens x 32 weight rows of fp32 results (lane l: row nrow0 + l,
// v[e] = token t0 + e) leave as 16-byte stores of 8 consecutive rows. Within each group of 8
// lanes the token-pair words go through an 8 x 8 transpose (3 shuffle stages: at stage b, lanes
// whose bit b differs swap the words whose index bit b differs from their own), after which lane
// i of group g holds tokens 2i and 2i+1 of rows 8g..8g+7 and writes each as one 16-byte store:
// 2 store instructions per 16 tokens instead of 16 of 4 bytes (with `add`, two 16-byte fp16 atomic
// adds). Needs N % 8 == 0 and nrow0 % 8 == 0.
__device__ __forceinline__ void store_rows16(const uint32_t (&v)[16], __half *C, int N, int M,
                                             int t0, int nrow0, int lane, bool add)
{
    uint32_t p[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        p[k] = pack_half2_rn(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
    const int i = lane & 7;
#pragma unroll
    for (int b = 4; b >= 1; b >>= 1) {
        const bool upper = (i & b) != 0;
#pragma unroll
        for (int k0 = 0; k0 < 8; ++k0) {
            if (k0 & b) continue;
            const int k1 = k0 | b;
            const uint32_t got = __shfl_xor_sync(0xffffffffu, upper ? p[k0] : p[k1], b);
            if (upper) p[k0] = got;
            else p[k1] = got;
        }
    }
    // p[j] = (token 2i, token 2i+1) of row j of the group
    const int n = nrow0 + 8 * (lane >> 3);
    const int ta = t0 + 2 * i;
    if (n < N) {
        const uint4 even = make_uint4(prmt_i<0x5410>(p[0], p[1]), prmt_i<0x5410>(p[2], p[3]),
                                      prmt_i<0x5410>(p[4], p[5]), prmt_i<0x5410>(p[6], p[7]));
        const uint4 odd = make_uint4(prmt_i<0x7632>(p[0], p[1]), prmt_i<0x7632>(p[2], p[3]),
                                     prmt_i<0x7632>(p[4], p[5]), prmt_i<0x7632>(p[6], p[7]));
        __half *c0 = C + (size_t)ta * N + n;
        if (add) {
            if (ta < M) red_add_f16x8(c0, even);
            if (ta + 1 < M) red_add_f16x8(c0 + N, odd);
        } else {
            if (ta < M) *reinterpret_cast<uint4 *>(c0) = even;
            if (ta + 1 < M) *reinterpret_cast<uint4 *>(c0 + N) = odd;
        }
    }
}

// Output tile of work unit u: units enumerate (split, token-tile group, weight tile, token tile).
struct Unit {
    int n0, t0, kb0, nk;
};

// kbps > 0: units are (K part of kbps slabs, tile). kbps < 0: stream-K schedule over the grid's G
// CTAs: the flattened (tile, copy of pg slabs) space is cut into G ranges of equal length, CTA c
// owning copies [c T / G, (c + 1) T / G); its range crosses at most J = -kbps tiles, and unit
// u = c + G j is the part of that range in the j-th of them (nk = 0 when there is none).
__device__ __forceinline__ Unit unit_of(int u, int n_tiles, int t_tiles, int BNv, int nkb,
                                        int kbps, int wr = kRowsW, int group_t = kGroupT,
                                        int pg = 1)
{
    const int tiles = n_tiles * t_tiles;
    int tile, kb0, nk;
    if (kbps < 0) {
        const int G = (int)gridDim.x, c = u % G, j = u / G;
        const int ncp = nkb / pg;
        const long long T = (long long)tiles * ncp;
        const long long a = (long long)c * T / G, b = (long long)(c + 1) * T / G;
        tile = (int)(a / ncp) + j;
        const long long s0 = max(a, (long long)tile * ncp), s1 = min(b, (long long)(tile + 1) * ncp);
        if (tile >= tiles || s0 >= s1) return Unit{0, 0, 0, 0};
        kb0 = (int)(s0 - (long long)tile * ncp) * pg;
        nk = (int)(s1 - s0) * pg;
    } else {
        const int split = u / tiles;
        tile = u - split * tiles;
        kb0 = split * kbps;
        nk = max(0, min(nkb, kb0 + kbps) - kb0);
    }
    const int per_group = group_t * n_tiles;
    const int group = tile / per_group;
    const int first_t = group * group_t;
    const int gt = min(group_t, t_tiles - first_t);
    const int within = tile - group * per_group;
    Unit w;
    w.t0 = (first_t + within % gt) * BNv;
    w.n0 = (within / gt) * wr;
    w.kb0 = kb0;
    w.nk = nk;
    return w;
}

// Persistent kernel: each CTA walks work units blockIdx.x, blockIdx.x + gridDim.x, ... The
// shared-memory ring runs on across units, and the accumulator is double-buffered in TMEM so the
// epilogue of one unit overlaps the main loop of the next (except in the 512-token tile, whose
// two accumulators fill TMEM: there the next unit's MMAs wait for the epilogue).
//   warps 0-3  epilogue (warp w reads TMEM lanes 32w..32w+31)
//   warp 4     TMA producer          warp 5  TMEM allocation + MMA issue
//   warp 6     TMA producer of packed weight slabs (packed formats)
//   warps 8-15 dequantisation of packed weights (two threads per weight row of the tile, or one
//              in the token-major variant)
// TOKA: token-major variant (W4A16): tiles of kTokT = BN tokens x kRowsT weight rows, tokens in
// the MMA's M, weights in its N; the accumulator holds one token per TMEM lane.
template <int MODE, int BN, int STAGES, int PG, bool TOKA, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
               const __half *__restrict__ S, const __half *__restrict__ Z, void *__restrict__ C,
               int M, int N, int K, int gs, int kb_per_split, int units, int atomic_out,
               const float *__restrict__ mult, unsigned int *err)
{
    using T = Traits<MODE>;
    using L = Smem<MODE, BN, STAGES, PG, TOKA, PAIR>;
    static_assert(!TOKA || (is_w4(MODE) && BN == kTokT), "token-major tiles: W4A16, 128 tokens");
    static_assert(!PAIR || (!TOKA && BN >= 128), "CTA pairs: weight-major tiles of 128+ tokens");
    constexpr int WR = L::WR;
    // DUAL (BN = 512, packed weights): each upcast weight slab feeds two MMAs, one per 256-token
    // half of the tile, into two accumulators that fill TMEM (no double buffering); the halves
    // arrive as consecutive activation stages
    constexpr bool DUAL = BN == 512;
    static_assert(!DUAL || (L::packed && !TOKA && !PAIR && STAGES % 2 == 0),
                  "512-token tiles: packed weights, weight-major, single CTA, even stages");
    constexpr int NH = DUAL ? 2 : 1;                  // activation stages per slab
    constexpr int BH = BN / NH;                       // tokens per activation stage
    constexpr int NMMA = TOKA ? kRowsT : BH;          // the MMA's N (accumulator columns)
    constexpr uint32_t kCols = DUAL ? 512u : tmem_cols<NMMA>();
    constexpr int NBUF = DUAL ? 1 : 2;                // accumulator buffers in TMEM
    constexpr int GT = DUAL ? kGroupT / 2 : kGroupT;  // token tiles per raster group
    constexpr uint32_t kIdesc = instr_desc<MODE, NMMA, PAIR ? 2 * kRowsW : kRowsW>();
    // CTA pairs: a unit covers UR = 256 weight rows, this CTA's 128 start at roff, and this CTA
    // loads tokens aoff .. aoff + AR - 1 of the tile; both CTAs walk the same units
    constexpr int UR = PAIR ? 2 * kRowsW : WR;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;
    const int roff = PAIR ? (int)rank * kRowsW : 0;
    const int aoff = PAIR ? (int)rank * L::AR : 0;
    const int ustart = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ustep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::bar_off);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + L::nbars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int n_tiles = (N + UR - 1) / UR;
    const int t_tiles = (M + BN - 1) / BN;
    const int nkb = (K + T::k_per_slab - 1) / T::k_per_slab;

    constexpr int DQ = L::dq, SP = L::sp;
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
    auto pfull_bar = [&](int p) { return smem_u32(bars + 2 * STAGES + p); };
    auto pempty_bar = [&](int p) { return smem_u32(bars + 2 * STAGES + SP + p); };
    auto dqf_bar = [&](int d) { return smem_u32(bars + 2 * STAGES + 2 * SP + d); };
    auto dqe_bar = [&](int d) { return smem_u32(bars + 2 * STAGES + 2 * SP + DQ + d); };
    auto accf_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 * SP + 2 * DQ + b); };
    auto acce_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 * SP + 2 * DQ + 2 + b); };
    const uint32_t final_bar = smem_u32(bars + 2 * STAGES + 2 * SP + 2 * DQ + 4);
    // dense / int8: stage s = [weight slab | activation slab]; packed: stage s = activation slab
    auto w_tma = [&](int s) { return base + s * (L::w_bytes + L::a_bytes); };
    auto a_tile = [&](int s) {
        return L::packed ? base + s * L::a_bytes : base + s * (L::w_bytes + L::a_bytes) + L::w_bytes;
    };
    auto pw_tile = [&](int p) { return base + L::pw_off + p * L::pw_bytes; };
    auto w_dq = [&](int d) { return base + L::dq_off + d * L::dq_bytes; };

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        // the 8 dequantisation warps arrive once each (lane 0, after __syncwarp): one arrival
        // per thread would serialise 256 shared-memory atomics on one barrier every slab
        for (int p = 0; p < SP; ++p) {
            mbar_init(pfull_bar(p), 1);
            mbar_init(pempty_bar(p), 8);
        }
        // a pair's leader hears the upcast and epilogue warps of both CTAs
        for (int d = 0; d < DQ; ++d) {
            mbar_init(dqf_bar(d), PAIR ? 16 : 8);
            mbar_init(dqe_bar(d), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), PAIR ? 8 : 4);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        if constexpr (PAIR) {
            // both CTAs of the pair, from the same warp, into the same shared-memory offset
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_holder)),
                         "r"(kCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(tmem_holder)),
                         "r"(kCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    // a pair's barriers must be initialised before the other CTA signals them
    if constexpr (PAIR) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // The producer and MMA warps run their loops with all 32 lanes, so that control flow, slot
    // indices, coordinates and descriptors stay warp-uniform: the compiler then keeps them in
    // uniform registers, which is where TMA and tcgen05.mma take their operands from (computed
    // in a one-lane branch they must be moved there first, which costs more than the issue
    // itself). Lane 0 issues; every lane waits, and the warp takes one decision per wait.
    if (warp == 4) {
        // ---------------- TMA producer (weight + activation slabs, or activations) --------
        constexpr uint32_t kTx = L::packed ? L::a_bytes : L::w_bytes + L::a_bytes;
        int it = 0;
        bool stop = false;
        for (int u = ustart; u < units && !stop; u += ustep) {
            const Unit w = unit_of(u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
            for (int i = 0; i < NH * w.nk; ++i, ++it) {
                const int s = it % STAGES;
                if (!warp_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1, abort_flag, err)) {
                    stop = true;
                    break;
                }
                // stage it holds K slab i / NH of tokens t0 + (i % NH) * BH .. + BH - 1
                const int kx = (w.kb0 + i / NH) * T::k_per_slab;
                const int ty = w.t0 + (i % NH) * BH;
                if (lane == 0) {
                    if constexpr (PAIR) {
                        // both CTAs' copies complete on the leader's barrier, which expects both
                        const uint32_t fb = map_to_rank(full_bar(s), 0);
                        if (rank == 0) mbar_expect_tx(full_bar(s), 2 * kTx);
                        if constexpr (!L::packed)
                            tma_load_2d_pair(smem_u32(w_tma(s)), &tm_w, fb, kx, w.n0 + roff);
                        tma_load_2d_pair(smem_u32(a_tile(s)), &tm_a, fb, kx, w.t0 + aoff);
                    } else if (DUAL && ty >= M) {
                        // a half with no tokens: no copy; its accumulator columns are never stored
                        mbar_arrive(full_bar(s));
                    } else {
                        mbar_expect_tx(full_bar(s), kTx);
                        if constexpr (!L::packed)
                            tma_load_2d(smem_u32(w_tma(s)), &tm_w, full_bar(s), kx, w.n0);
                        tma_load_2d(smem_u32(a_tile(s)), &tm_a, full_bar(s), kx, ty);
                    }
                }
                __syncwarp();
            }
        }
        // every copy this warp started must land before the CTA can exit
        if (!PAIR || rank == 0) {
            for (int i = max(0, it - STAGES); i < it; ++i) {
                int dummy_abort = 0;
                mbar_wait(full_bar(i % STAGES), (i / STAGES) & 1, &dummy_abort, nullptr);
            }
        } else if (*abort_flag) {
            // the second CTA's copies complete on the leader's barrier, which it cannot watch:
            // after a give-up (the only way it can stop early) it waits 100 us, far beyond the
            // latency of a copy, before it heads for the exit
            const uint64_t t0 = global_ns();
            while (global_ns() - t0 < 100000ull) __nanosleep(1000);
        }
    } else if (warp == 6) {
        if constexpr (L::packed) {
            // ---------------- TMA producer (packed weight slabs) ----------------
            int it = 0;
            bool stop = false;
            for (int u = ustart; u < units && !stop; u += ustep) {
                const Unit w = unit_of(u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
                // units cover whole copies: with PG > 1 the split and K are multiples of PG slabs
                for (int i = 0; i < w.nk; i += PG, ++it) {
                    const int p = it % SP;
                    if (!warp_wait(pempty_bar(p), ((it / SP) & 1) ^ 1, abort_flag, err)) {
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        mbar_expect_tx(pfull_bar(p), L::pw_bytes);
                        tma_load_2d(smem_u32(pw_tile(p)), &tm_w, pfull_bar(p), (w.kb0 + i) * 8,
                                    w.n0 + roff);
                    }
                    __syncwarp();
                }
            }
            for (int i = max(0, it - SP); i < it; ++i) {
                int dummy_abort = 0;
                mbar_wait(pfull_bar(i % SP), (i / SP) & 1, &dummy_abort, nullptr);
            }
        }
    } else if (warp == 5 && (!PAIR || rank == 0)) {
        // ---------------- MMA issuer (a pair's leader issues for both CTAs) ----------------
        // Lane 0 issues the MMAs and the commits: a commit tracks the MMAs its own thread issued.
        int it = 0, sa = 0, j = 0;   // slabs, activation stages and units consumed
        bool stop = false;
        for (int u = ustart; u < units && !stop; u += ustep) {
            const Unit w = unit_of(u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
            if (w.nk == 0) continue;
            const int b = NBUF == 2 ? j & 1 : 0;
            const int use = NBUF == 2 ? j >> 1 : j;     // earlier uses of buffer b
            if (!warp_wait(acce_bar(b), (use & 1) ^ 1, abort_flag, err)) break;
            tc_fence_after();
            const uint32_t dtm = tmem_base + (uint32_t)(b * NMMA);
            // one slab at a time: wait for its activation stage (and upcast weights), issue its 4
            // MMAs, then commit its buffers back at once, so that every buffer returns to its
            // producer as soon as the tensor core is done with it (a commit tracks all MMAs this
            // thread issued before it)
            for (int i = 0; i < w.nk; ++i, ++it, sa += NH) {
                const int s = sa % STAGES;
                const int d = T::packed ? it % DQ : 0;
                bool ready = true;
                if constexpr (T::packed) ready = warp_wait(dqf_bar(d), (it / DQ) & 1, abort_flag, err);
#pragma unroll
                for (int h = 0; h < NH; ++h)
                    ready = ready && warp_wait(full_bar((sa + h) % STAGES), ((sa + h) / STAGES) & 1,
                                               abort_flag, err);
                if (!ready) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if constexpr (DUAL) {
                    // the upcast slab against both 256-token halves: 4 MMAs into each accumulator,
                    // each half's activation stage released once its MMAs are done
                    const uint64_t wdesc = sw128_desc(smem_u32(w_dq(d)));
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            const int sh = (sa + h) % STAGES;
                            const uint64_t tdesc = sw128_desc(smem_u32(a_tile(sh)));
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                mma_issue<MODE>(dtm + (uint32_t)(h * BH), wdesc + 2 * k, tdesc + 2 * k,
                                                kIdesc, (i | k) != 0 ? 1u : 0u);
                            mma_commit(empty_bar(sh));
                        }
                        mma_commit(dqe_bar(d));
                    }
                    __syncwarp();
                    continue;
                }
                const uint64_t wdesc = sw128_desc(smem_u32(T::packed ? w_dq(d) : w_tma(s)));
                const uint64_t tdesc = sw128_desc(smem_u32(a_tile(s)));
                const uint64_t adesc = TOKA ? tdesc : wdesc, bdesc = TOKA ? wdesc : tdesc;
                if (lane == 0) {
                    if constexpr (PAIR) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_issue_pair<MODE>(dtm, adesc + 2 * k, bdesc + 2 * k, kIdesc,
                                                 (i | k) != 0 ? 1u : 0u);
                        // the slab's buffers go back to their producers in both CTAs
                        mma_commit_pair_both(empty_bar(s));
                        if constexpr (T::packed) mma_commit_pair_both(dqe_bar(d));
                    } else {
#pragma unroll
                        for (int k = 0; k < 4; ++k)   // 4 MMAs of 32 bytes of K each
                            mma_issue<MODE>(dtm, adesc + 2 * k, bdesc + 2 * k, kIdesc,
                                            (i | k) != 0 ? 1u : 0u);
                        mma_commit(empty_bar(s));
                        if constexpr (T::packed) mma_commit(dqe_bar(d));
                    }
                }
                __syncwarp();
            }
            if (stop) break;
            if (lane == 0) {
                if constexpr (PAIR) mma_commit_pair_both(accf_bar(b));
                else mma_commit(accf_bar(b));
            }
            __syncwarp();
            ++j;
        }
        // nothing may still run on the tensor cores when TMEM is released
        if (lane == 0) {
            if constexpr (PAIR) mma_commit_pair_local(final_bar);
            else mma_commit(final_bar);
        }
        __syncwarp();
        int dummy_abort = 0;
        mbar_wait(final_bar, 0, &dummy_abort, nullptr);
    } else if (warp >= 8) {
        // ---------------- dequantisation (packed weights) ----------------
        // 256 threads: thread (h, r) upcasts words 4h..4h+3 of weight row r of every slab. The
        // scale and zero of the next slab are loaded while the current one is processed.
        if constexpr (T::packed) {
            const int dq = tid - 256;
            // thread (h, r) upcasts half h of weight row r; in the token-major variant thread r
            // upcasts both halves of row r (h = 0 then names the slab's scale group: the group
            // size is a multiple of 64 there)
            constexpr int NH = TOKA ? 2 : 1;
            const int r = TOKA ? dq : (dq & 127), h = TOKA ? 0 : (dq >> 7);
            volatile uint32_t *sink = reinterpret_cast<volatile uint32_t *>(base + L::sink_off);
            const int G = K / gs;
            // cursor over this CTA's slabs: unit u (position i inside it, w its coordinates)
            struct Cursor {
                int u, i;
                Unit w;
            };
            auto settle = [&](Cursor &c) {
                while (c.u < units && c.i >= c.w.nk) {
                    c.u += ustep;
                    c.i = 0;
                    if (c.u < units) c.w = unit_of(c.u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
                }
            };
            Cursor cur{ustart, 0, unit_of(ustart, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG)};
            settle(cur);
            // Scales and zeros. Per slab a thread needs s[n][g] and z[n][g] of its row n. Loading
            // those 2-byte values one slab at a time makes every warp touch 32 rows (32 sectors)
            // per load, which saturates the LSU. Instead each thread keeps a window of 8
            // consecutive groups of its row in registers (one 16-byte load for s, one for z) and
            // prefetches the following window while it works through the current one. This needs
            // G % 8 == 0 and 16-byte aligned scale / zero arrays; otherwise the values are
            // loaded per slab, kLook slabs ahead.
            const bool windowed = is_w4(MODE) && G % 8 == 0 &&
                                  (reinterpret_cast<uintptr_t>(S) & 15) == 0 &&
                                  (reinterpret_cast<uintptr_t>(Z) & 15) == 0;
            // group of a thread's half slab; a shift when the group size is a power of two
            const int gs_shift = (gs & (gs - 1)) == 0 ? __ffs(gs) - 1 : -1;
            auto group_of = [&](const Cursor &c) {
                const int k = (c.w.kb0 + c.i) * 64 + 32 * h;
                return min(gs_shift >= 0 ? k >> gs_shift : k / gs, G - 1);
            };
            struct Window {
                int u, gb;                 // unit and first group (multiple of 8); u < 0: none
                uint4 s, z;                // fp16 s and z of groups gb .. gb+7 of this row
            };
            auto load_window = [&](Window &wnd, int u, const Unit &w, int gb) {
                wnd.u = u;
                wnd.gb = gb;
                if (u >= units) return;
                const size_t off = (size_t)min(w.n0 + roff + r, N - 1) * G + gb;
                wnd.s = ld_cached_v4(S + off);
                wnd.z = Z ? ld_cached_v4(Z + off) : make_uint4(0u, 0u, 0u, 0u);
            };
            // the window after wnd in this CTA's walk (same unit, or the next unit's first one)
            auto next_window = [&](Window &out, const Window &wnd) {
                const Unit w = unit_of(wnd.u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
                const int g_last = min(((w.kb0 + w.nk) * 64 - 1) / gs, G - 1);
                if (wnd.gb + 8 <= g_last) {
                    load_window(out, wnd.u, w, wnd.gb + 8);
                    return;
                }
                int u = wnd.u + ustep;
                Unit nw = w;
                while (u < units) {
                    nw = unit_of(u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
                    if (nw.nk > 0) break;
                    u += ustep;
                }
                load_window(out, u, nw, (min((nw.kb0 * 64) / gs, G - 1)) & ~7);
            };
            // the current window as fp16 pairs ready for the upcast: s and fp16(-z * s)
            uint4 win_s = make_uint4(0u, 0u, 0u, 0u), win_nz = make_uint4(0u, 0u, 0u, 0u);
            auto make_current = [&](const Window &wnd) {
                const uint32_t sv[4] = {wnd.s.x, wnd.s.y, wnd.s.z, wnd.s.w};
                const uint32_t zv[4] = {wnd.z.x, wnd.z.y, wnd.z.z, wnd.z.w};
                uint32_t nz[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 sf = __half22float2(*reinterpret_cast<const __half2 *>(&sv[q]));
                    const float2 zf = __half22float2(*reinterpret_cast<const __half2 *>(&zv[q]));
                    nz[q] = pack_half2_rn(-zf.x * sf.x, -zf.y * sf.y);
                }
                win_s = wnd.s;
                win_nz = make_uint4(nz[0], nz[1], nz[2], nz[3]);
            };
            // element j (0..7) of v, duplicated into both halves
            auto pick2 = [](const uint4 &v, int j) {
                const uint32_t lo = (j & 2) ? v.y : v.x, hi = (j & 2) ? v.w : v.z;
                const uint32_t wv = (j & 4) ? hi : lo;
                return prmt(wv, wv, (j & 1) ? 0x3232u : 0x1010u);
            };
            Window wcur{-1, 0, {}, {}}, wnxt{-1, 0, {}, {}};
            if (windowed && cur.u < units) {
                load_window(wcur, cur.u, cur.w, group_of(cur) & ~7);
                make_current(wcur);
                next_window(wnxt, wcur);
            }
            // per-slab fallback: scale and zero loaded kLook slabs ahead
            constexpr int kLook = 4;
            float sc[kLook], zz[kLook];
            Cursor ahead = cur;
            auto fetch = [&](const Cursor &c, float &s_out, float &z_out) {
                if (!is_w4(MODE) || windowed || c.u >= units) {
                    s_out = 0.f;
                    z_out = 0.f;
                    return;
                }
                const int n = min(c.w.n0 + roff + r, N - 1);
                const int g = group_of(c);
                s_out = half_bits_to_float(ld_cached_u16(S + (size_t)n * G + g));
                z_out = Z ? half_bits_to_float(ld_cached_u16(Z + (size_t)n * G + g)) : 0.f;
            };
#pragma unroll
            for (int q = 0; q < kLook; ++q) {
                fetch(ahead, sc[q], zz[q]);
                ++ahead.i;
                settle(ahead);
            }
            // scale and zero of the slab at cur as fp16 pairs (s, s) and (-z s, -z s); advances
            // the scale window or the look-ahead of the per-slab fallback
            auto slab_scales = [&](uint32_t &sc2, uint32_t &nz2) {
                sc2 = 0u;
                nz2 = 0u;
                if (windowed) {
                    const int g = group_of(cur);
                    if (wcur.u != cur.u || g < wcur.gb || g >= wcur.gb + 8) {
                        if (wnxt.u == cur.u && g >= wnxt.gb && g < wnxt.gb + 8) wcur = wnxt;
                        else load_window(wcur, cur.u, cur.w, g & ~7);
                        make_current(wcur);
                        next_window(wnxt, wcur);
                    }
                    sc2 = pick2(win_s, g - wcur.gb);
                    nz2 = pick2(win_nz, g - wcur.gb);
                } else if (is_w4(MODE)) {
                    sc2 = half2_bcast(sc[0]);
                    nz2 = half2_bcast(-zz[0] * sc[0]);
#pragma unroll
                    for (int q = 0; q + 1 < kLook; ++q) {   // shift the window (static indices)
                        sc[q] = sc[q + 1];
                        zz[q] = zz[q + 1];
                    }
                    fetch(ahead, sc[kLook - 1], zz[kLook - 1]);
                    ++ahead.i;
                    settle(ahead);
                }
            };
            // one packed copy (PG slabs) per iteration: the copy's loads are issued together, its
            // slabs upcast one after another, each into the next free upcast buffer
            int it = 0;
            while (cur.u < units) {
                uint32_t sc2[PG], nz2[PG];
#pragma unroll
                for (int j = 0; j < PG; ++j) {
                    slab_scales(sc2[j], nz2[j]);
                    if (j + 1 < PG) ++cur.i;   // a copy never straddles units
                }
                const int pc = it / PG, pp = pc % SP;
                // waits decide for the whole warp: the warp-level hand-overs below need all lanes
                if (!warp_wait(pfull_bar(pp), (pc / SP) & 1, abort_flag, err)) break;
                uint4 pk[PG][NH];
#pragma unroll
                for (int j = 0; j < PG; ++j)
#pragma unroll
                    for (int x = 0; x < NH; ++x) {
                        const int hv = TOKA ? x : h;
                        if constexpr (PG == 1) {
                            const uint32_t *packed = reinterpret_cast<const uint32_t *>(pw_tile(pp));
                            pk[j][x] = *reinterpret_cast<const uint4 *>(packed + r * 8 +
                                                                        4 * (hv ^ ((r >> 2) & 1)));
                        } else {
                            // 128-byte rows under the 128-byte swizzle: 16-byte piece c of row r
                            // sits at c ^ (r & 7); slab j's half h is piece 2 j + h
                            pk[j][x] = *reinterpret_cast<const uint4 *>(
                                pw_tile(pp) + r * 128 + 16 * ((2 * j + hv) ^ (r & 7)));
                        }
                    }
                // The slot goes back to the TMA producer only once every lane's loads of it have
                // returned: an arrival does not wait for loads still in flight in other lanes, and
                // the next copy into the slot would overwrite data not yet read. A store of a
                // value computed from all four loads cannot issue before they return, and the
                // arrival (a release) is ordered after it.
                uint32_t landed = 0;
#pragma unroll
                for (int j = 0; j < PG; ++j)
#pragma unroll
                    for (int x = 0; x < NH; ++x)
                        landed ^= pk[j][x].x ^ pk[j][x].y ^ pk[j][x].z ^ pk[j][x].w;
                sink[dq] = landed;
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty_bar(pp));   // the packed copy is read in full
                bool ok = true;
#pragma unroll
                for (int j = 0; j < PG; ++j) {
                    const int d = (it + j) % DQ;
                    if (!warp_wait(dqe_bar(d), (((it + j) / DQ) & 1) ^ 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int x = 0; x < NH; ++x) {
                        if constexpr (is_w4(MODE))
                            dequant_w4<MODE == kW4A16I>(pk[j][x], w_dq(d), r, TOKA ? x : h, sc2[j],
                                                        nz2[j]);
                        else
                            dequant_w2<MODE == kW2A8I>(pk[j][x], w_dq(d), r, h);
                    }
                    if constexpr (per_slab_handoff(BN)) {
                        // this slab's upcast stores become visible to the tensor core (async
                        // proxy), then one arrival per warp hands the buffer over (to the
                        // pair's leader, which issues the MMA)
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(dqf_bar(d), 0));
                            else mbar_arrive(dqf_bar(d));
                        }
                    }
                }
                if (!ok) break;
                if constexpr (!per_slab_handoff(BN)) {
                    // the same for the whole copy: one fence, then the PG buffers in order
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
#pragma unroll
                        for (int j = 0; j < PG; ++j) {
                            if constexpr (PAIR)
                                mbar_arrive_cluster(map_to_rank(dqf_bar((it + j) % DQ), 0));
                            else
                                mbar_arrive(dqf_bar((it + j) % DQ));
                        }
                }
                it += PG;
                ++cur.i;
                settle(cur);
            }
        }
    } else if (warp < 4) {
        // ---------------- epilogue ----------------
        const int r = tid;                                 // weight row of the tile = TMEM lane
        const bool pairs = (N & 1) == 0;
        int j = 0;
        for (int u = ustart; u < units; u += ustep) {
            const Unit w = unit_of(u, n_tiles, t_tiles, BN, nkb, kb_per_split, UR, GT, PG);
            if (w.nk == 0) continue;
            const int b = NBUF == 2 ? j & 1 : 0;
            bool ok = mbar_wait(accf_bar(b), (NBUF == 2 ? j >> 1 : j) & 1, abort_flag, err);
            tc_fence_after();
            // tcgen05.ld is warp-collective: decide per warp, never per lane
            ok = __all_sync(0xffffffffu, ok && !*abort_flag);
            if (!ok) break;
            if constexpr (TOKA) {
                // token-major: TMEM lane = token, columns = the tile's 256 weight rows, so each
                // thread's results are contiguous in C (row t); tcgen05.ld stays warp-wide
                const int t = w.t0 + tid;
                const uint32_t lane_addr =
                    tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * NMMA);
                const bool vec16 = (N & 7) == 0;
                if (w.t0 + warp * 32 < M) {
#pragma unroll 1
                    for (int c = 0; c < NMMA; c += 16) {
                        const int n = w.n0 + c;
                        if (n >= N) break;
                        uint32_t v[16];
                        tmem_ld16(lane_addr + c, v);
                        if (t >= M) continue;
                        __half *dst = static_cast<__half *>(C) + (size_t)t * N + n;
                        uint32_t h2[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            h2[i] = pack_half2_rn(__uint_as_float(v[2 * i]),
                                                  __uint_as_float(v[2 * i + 1]));
                        if (n + 16 <= N && pairs) {
                            if (atomic_out && vec16) {
                                red_add_f16x8(dst, make_uint4(h2[0], h2[1], h2[2], h2[3]));
                                red_add_f16x8(dst + 8, make_uint4(h2[4], h2[5], h2[6], h2[7]));
                            } else if (atomic_out) {
#pragma unroll
                                for (int i = 0; i < 8; ++i) red_add_f16x2(dst + 2 * i, h2[i]);
                            } else if (vec16) {
                                reinterpret_cast<uint4 *>(dst)[0] = make_uint4(h2[0], h2[1], h2[2], h2[3]);
                                reinterpret_cast<uint4 *>(dst)[1] = make_uint4(h2[4], h2[5], h2[6], h2[7]);
                            } else {
#pragma unroll
                                for (int i = 0; i < 8; ++i) reinterpret_cast<uint32_t *>(dst)[i] = h2[i];
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                if (n + e >= N) break;
                                const float x = __uint_as_float(v[e]);
                                if (atomic_out) red_add_f16(dst + e, half_bits_rn(x));
                                else dst[e] = __float2half_rn(x);
                            }
                        }
                    }
                }
            } else {
                const int n = w.n0 + roff + r;
                // fp16 results leave as 16-byte stores (or 16-byte atomic adds) of 8 rows
                const bool rows16 = (N & 7) == 0;
                // int8 requantisation (int32 modes): this lane's output-channel multiplier
                const float rq = (T::c_bytes == 4 && mult && n < N) ? mult[n] : 0.f;
                const uint32_t lane_addr =
                    tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * BN);
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    if (w.t0 + c >= M) break;
                    uint32_t v[16];
                    tmem_ld16(lane_addr + c, v);
                    if constexpr (T::c_bytes == 2) {
                        if (rows16) {
                            store_rows16(v, static_cast<__half *>(C), N, M, w.t0 + c,
                                         w.n0 + roff + 32 * warp, lane, atomic_out != 0);
                            continue;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int t = w.t0 + c + e;           // the same in every lane
                        if (t >= M) break;
                        if constexpr (T::c_bytes == 2) {
                            // fp16 results leave as (n, n+1) pairs from neighbouring lanes
                            const float x = __uint_as_float(v[e]);
                            const float y = __shfl_xor_sync(0xffffffffu, x, 1);
                            __half *dst = static_cast<__half *>(C) + (size_t)t * N + n;
                            if (pairs) {
                                if ((lane & 1) == 0 && n < N) {
                                    const uint32_t h2 = pack_half2_rn(x, y);
                                    if (atomic_out) red_add_f16x2(dst, h2);
                                    else *reinterpret_cast<uint32_t *>(dst) = h2;
                                }
                            } else if (n < N) {
                                if (atomic_out) red_add_f16(dst, half_bits_rn(x));
                                else *dst = __float2half_rn(x);
                            }
                        } else if (n < N) {
                            const size_t idx = (size_t)t * N + n;
                            if (mult) static_cast<int8_t *>(C)[idx] = requant_i8((int)v[e], rq);
                            else if (atomic_out) red_add_s32(static_cast<int32_t *>(C) + idx, (int)v[e]);
                            else static_cast<int32_t *>(C)[idx] = (int)v[e];
                        }
                    }
                }
            }
            // this warp is done with accumulator buffer b (the pair's leader waits for both CTAs)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(map_to_rank(acce_bar(b), 0));
                else mbar_arrive(acce_bar(b));
            }
            ++j;
        }
    }

    tc_fence_before();
    // a pair: the leader's last MMA (waited for above) read the other CTA's shared memory and
    // wrote its TMEM, so neither CTA releases anything before both are here
    if constexpr (PAIR) cluster_sync();
    else __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(kCols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(kCols)
                         : "memory");
    }
}

// ---- host side -----------------------------------------------------------------------------------

int mode_of(int op)
{
    switch (op) {
    case QG_OP_DENSE_F16: return kDense;
    case QG_OP_W8A8: return kW8A8;
    case QG_OP_W4A16: return kW4A16;
    default: return kW2A8;
    }
}

// pair: a CTA pair shares the tile (each CTA holds half of the token rows of a stage)
int smem_bytes(int mode, int bn, int stages, int pg, int wr = kRowsW, bool pair = false)
{
    const bool packed = (is_w4(mode) || mode == kW2A8);
    const int ar = act_rows(bn, pair);
    return smem_total(packed, ar, stages, dq_buffers(packed, bn, stages, pg, wr, ar), pg,
                      packed ? packed_stages(pg, bn, stages, wr, ar) : 0, wr);
}

// slabs per packed-weight copy for this problem and tile: 4 when K holds a whole number of
// 4-slab runs and that plan fits in shared memory, else 1
int packed_group(const Problem &p, int bn, int stages, int wr = kRowsW, bool pair = false)
{
    const int mode = mode_of(p.op);
    if (!(is_w4(mode) || mode == kW2A8)) return 1;
    const int kps = is_w4(mode) ? 64 : 128;
    if (p.K % kps || (p.K / kps) % 4) return 1;
    return smem_bytes(mode, bn, stages, 4, wr, pair) <= kMaxSmem ? 4 : 1;
}

// streamk: the stream-K schedule (every CTA gets an equal share of the (tile, K) work; partial
// tiles are added into the zeroed output)
template <int MODE, int BN, int STAGES, int PG, bool TOKA = false, bool PAIR = false>
cudaError_t launch_t(const Problem &p, int split_k, unsigned int *err, cudaStream_t stream,
                     bool streamk = false)
{
    using T = Traits<MODE>;
    using L = Smem<MODE, BN, STAGES, PG, TOKA, PAIR>;
    if (L::total > kMaxSmem) return cudaErrorInvalidConfiguration;
    auto kern = tc_gemm_kernel<MODE, BN, STAGES, PG, TOKA, PAIR>;
    // the dynamic shared-memory opt-in is per device: remember it per device
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
    bool ok;
    if constexpr (MODE == kDense) {
        ok = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.W, p.K, p.N, (uint64_t)p.K * 2, 64,
                      kRowsW, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.A, p.K, p.M, (uint64_t)p.K * 2, 64,
                      L::AR, CU_TENSOR_MAP_SWIZZLE_128B);
    } else if constexpr (MODE == kW8A8) {
        ok = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.W, p.K, p.N, (uint64_t)p.K, 128,
                      kRowsW, CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.A, p.K, p.M, (uint64_t)p.K, 128, L::AR,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    } else if constexpr (is_w4(MODE)) {
        ok = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, p.K / 8, p.N, (uint64_t)p.K / 2,
                      8 * PG, L::WR, PG == 1 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.A, p.K, p.M, (uint64_t)p.K * 2, 64,
                      L::AR, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, p.K / 16, p.N, (uint64_t)p.K / 4,
                      8 * PG, kRowsW, PG == 1 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.A, p.K, p.M, (uint64_t)p.K, 128, L::AR,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) return cudaErrorInvalidValue;

    const int nkb = (p.K + T::k_per_slab - 1) / T::k_per_slab;
    const int kbps = ((nkb + split_k - 1) / split_k + PG - 1) / PG * PG;   // whole copies
    const int splits = (nkb + kbps - 1) / kbps;
    constexpr int UR = PAIR ? 2 * kRowsW : L::WR;      // weight rows per unit
    const int n_tiles = (p.N + UR - 1) / UR;
    const int t_tiles = (p.M + BN - 1) / BN;
    long units = (long)n_tiles * t_tiles * splits;
    if (units > 0x7fffffffL) return cudaErrorInvalidValue;
    if (streamk && (PAIR || nkb % PG)) return cudaErrorInvalidValue;
    // persistent grid: as many CTAs (CTA pairs) as fit on the device at once (shared memory,
    // threads and the TMEM columns each CTA holds), never more than there are units
    static int per_dev[64] = {};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::total;
    cfg.stream = stream;
    if constexpr (PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (!per_dev[dev]) {
        int resident = 0;
        if constexpr (PAIR) {
            // clusters of two that fit at once (one CTA per SM: the kernel holds all of TMEM's
            // columns at 256 tokens and most of shared memory)
            cfg.gridDim = dim3(2);
            if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess)
                return cudaErrorInvalidConfiguration;
        } else {
            int occ = 0, sms = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, L::total) !=
                    cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return cudaErrorInvalidConfiguration;
            occ = std::min(occ, BN > 256 ? 1 : (int)(512 / tmem_cols<TOKA ? kRowsT : BN>()));
            resident = std::max(1, occ) * sms;
        }
        if (resident <= 0) return cudaErrorInvalidConfiguration;
        per_dev[dev] = resident;
    }
    int kb_arg = kbps;
    if (streamk) {
        // G CTAs, each owning ceil(T / G) copies at most, which cross at most J tiles
        const long G = per_dev[dev], ncp = nkb / PG, T = (long)n_tiles * t_tiles * ncp;
        const long J = ((T + G - 1) / G + ncp - 1) / ncp + 1;
        units = G * J;
        if (units > 0x7fffffffL) return cudaErrorInvalidValue;
        kb_arg = -(int)J;
    }
    const int slots = (int)std::min<long>(units, (long)per_dev[dev]);
    cfg.gridDim = dim3(PAIR ? 2 * slots : slots);
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, kern, tw, ta, static_cast<const __half *>(p.scales),
        p.has_zero ? static_cast<const __half *>(p.zeros) : nullptr, p.C, p.M, p.N, p.K, p.gs,
        kb_arg, (int)units, (split_k > 1 || streamk) ? 1 : 0, p.mult, err);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int MODE, int BN, int PG>
cudaError_t launch_stages_pg(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                             cudaStream_t stream)
{
    switch (c.stages) {
    case 2: return launch_t<MODE, BN, 2, PG>(p, c.split_k, err, stream, c.rows == 1);
    case 3: return launch_t<MODE, BN, 3, PG>(p, c.split_k, err, stream, c.rows == 1);
    case 4: return launch_t<MODE, BN, 4, PG>(p, c.split_k, err, stream, c.rows == 1);
    case 5: return launch_t<MODE, BN, 5, PG>(p, c.split_k, err, stream, c.rows == 1);
    default: break;
    }
    // deep activation rings for small token tiles: a small activation copy waits ~2-3 us behind
    // the weight stream, so only many stages in flight keep the MMA fed
    if constexpr (BN <= 128)
        if (c.stages == 8) return launch_t<MODE, BN, 8, PG>(p, c.split_k, err, stream, c.rows == 1);
    if constexpr (BN <= 64)
        if (c.stages == 16) return launch_t<MODE, BN, 16, PG>(p, c.split_k, err, stream, c.rows == 1);
    return cudaErrorInvalidValue;
}

template <int MODE, int BN>
cudaError_t launch_stages(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                          cudaStream_t stream)
{
    if constexpr (is_w4(MODE) || is_w2(MODE))
        if (packed_group(p, BN, c.stages) == 4) return launch_stages_pg<MODE, BN, 4>(p, c, err, stream);
    return launch_stages_pg<MODE, BN, 1>(p, c, err, stream);
}

// token-major variant (swap_ab = 0): tiles of 128 tokens x 256 weight rows, W4A16 only
template <int MODE>
cudaError_t launch_toka(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                        cudaStream_t stream)
{
    const bool g4 = packed_group(p, kTokT, c.stages, kRowsT) == 4;
    switch (c.stages) {
    case 2: return g4 ? launch_t<MODE, kTokT, 2, 4, true>(p, c.split_k, err, stream, c.rows == 1)
                      : launch_t<MODE, kTokT, 2, 1, true>(p, c.split_k, err, stream, c.rows == 1);
    case 3: return g4 ? launch_t<MODE, kTokT, 3, 4, true>(p, c.split_k, err, stream, c.rows == 1)
                      : launch_t<MODE, kTokT, 3, 1, true>(p, c.split_k, err, stream, c.rows == 1);
    case 4: return g4 ? launch_t<MODE, kTokT, 4, 4, true>(p, c.split_k, err, stream, c.rows == 1)
                      : launch_t<MODE, kTokT, 4, 1, true>(p, c.split_k, err, stream, c.rows == 1);
    default: return cudaErrorInvalidValue;
    }
}

// CTA pairs (bm = 256): weight-major tiles of 256 weight rows x BN tokens shared by two SMs
// (grouped packed copies only)
template <int MODE, int BN>
cudaError_t launch_pair(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                        cudaStream_t stream)
{
    constexpr int PG = (is_w4(MODE) || is_w2(MODE)) ? 4 : 1;
    switch (c.stages) {
    case 3: return launch_t<MODE, BN, 3, PG, false, true>(p, c.split_k, err, stream);
    case 4: return launch_t<MODE, BN, 4, PG, false, true>(p, c.split_k, err, stream);
    case 5: return launch_t<MODE, BN, 5, PG, false, true>(p, c.split_k, err, stream);
    case 8: return launch_t<MODE, BN, 8, PG, false, true>(p, c.split_k, err, stream);
    default: return cudaErrorInvalidValue;
    }
}

// 512-token weight-major tiles (packed weights): two 256-token accumulators fed by each upcast
// slab, activation stages in pairs
template <int MODE>
cudaError_t launch_dual(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                        cudaStream_t stream)
{
    if constexpr (is_w4(MODE) || is_w2(MODE)) {
        const bool g4 = packed_group(p, 512, c.stages) == 4;
        switch (c.stages) {
        case 2: return g4 ? launch_t<MODE, 512, 2, 4>(p, c.split_k, err, stream, c.rows == 1)
                          : launch_t<MODE, 512, 2, 1>(p, c.split_k, err, stream, c.rows == 1);
        case 4: return g4 ? launch_t<MODE, 512, 4, 4>(p, c.split_k, err, stream, c.rows == 1)
                          : launch_t<MODE, 512, 4, 1>(p, c.split_k, err, stream, c.rows == 1);
        default: break;
        }
    }
    return cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_bn(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream)
{
    if (c.bm == 2 * kRowsW) {
        if (c.bn == 128) return launch_pair<MODE, 128>(p, c, err, stream);
        if (c.bn == 256) return launch_pair<MODE, 256>(p, c, err, stream);
        return cudaErrorInvalidValue;
    }
    switch (c.bn) {
    case 16: return launch_stages<MODE, 16>(p, c, err, stream);
    case 32: return launch_stages<MODE, 32>(p, c, err, stream);
    case 64: return launch_stages<MODE, 64>(p, c, err, stream);
    case 128: return launch_stages<MODE, 128>(p, c, err, stream);
    case 256: return launch_stages<MODE, 256>(p, c, err, stream);
    case 512: return launch_dual<MODE>(p, c, err, stream);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace

bool tc_supports(const Problem &p, const qgemm_config_t &c)
{
    if (c.path != QG_PATH_TC) return false;
    // rows = 1: the stream-K schedule (single-CTA tiles, results added into the zeroed output:
    // not for the requantised int8 output, which needs whole sums)
    if (c.rows != 0 && c.rows != 1) return false;
    if (c.rows == 1 && (c.bm == 2 * kRowsW || c.split_k != 1 || p.mult)) return false;
    if (!c.swap_ab) {
        // token-major variant: W4A16 with scale groups of whole slabs
        if (p.op != QG_OP_W4A16 || c.bm != kTokT || c.bn != kRowsT) return false;
        if (c.stages < 2 || c.stages > 4 || c.split_k < 1 || c.split_k > 64) return false;
        if (p.K % 64 || p.gs % 64 || p.K % p.gs) return false;
        const int pg = packed_group(p, kTokT, c.stages, kRowsT);
        return smem_bytes(kW4A16, kTokT, c.stages, pg, kRowsT) <= kMaxSmem &&
               dq_buffers(true, kTokT, c.stages, pg, kRowsT) >= 3;
    }
    if (c.split_k < 1 || c.split_k > 64) return false;
    if (c.bm == 2 * kRowsW) {
        // CTA pair: 256 weight rows x 128 / 256 tokens, each CTA holding half of the tokens
        const int mode = mode_of(p.op);
        const bool packed = is_w4(mode) || mode == kW2A8;
        if (c.bn != 128 && c.bn != 256) return false;
        if (c.stages != 3 && c.stages != 4 && c.stages != 5 && c.stages != 8) return false;
        if (packed && packed_group(p, c.bn, c.stages, kRowsW, true) != 4) return false;
        if (smem_bytes(mode, c.bn, c.stages, packed ? 4 : 1, kRowsW, true) > kMaxSmem) return false;
        if (packed && dq_buffers(true, c.bn, c.stages, 4, kRowsW, c.bn / 2) < want_dq(4, c.bn))
            return false;
    } else if (c.bn == 512) {
        // two 256-token accumulators per upcast slab: packed weights, activation stages in pairs
        const int mode = mode_of(p.op);
        if (!(is_w4(mode) || mode == kW2A8)) return false;
        if (c.bm != 0 && c.bm != kRowsW) return false;
        if (c.stages != 2 && c.stages != 4) return false;
        const int pg = packed_group(p, 512, c.stages);
        if (smem_bytes(mode, 512, c.stages, pg) > kMaxSmem) return false;
        if (dq_buffers(true, 512, c.stages, pg, kRowsW, 256) < want_dq(pg, 512)) return false;
    } else {
        if (c.bm != 0 && c.bm != kRowsW) return false;
        if (c.bn != 16 && c.bn != 32 && c.bn != 64 && c.bn != 128 && c.bn != 256) return false;
        if (!((c.stages >= 2 && c.stages <= 5) || (c.bn <= 128 && c.stages == 8) ||
              (c.bn <= 64 && c.stages == 16)))
            return false;
        if (smem_bytes(mode_of(p.op), c.bn, c.stages, packed_group(p, c.bn, c.stages)) > kMaxSmem)
            return false;
    }
    if (p.op == QG_OP_W4A16 && (p.K % 32 || p.gs % 32 || p.K % p.gs)) return false;
    if (p.op == QG_OP_W2A8 && p.K % 64) return false;
    if (p.op == QG_OP_W8A8 && p.K % 16) return false;
    if (p.op == QG_OP_DENSE_F16 && p.K % 8) return false;
    return true;
}

int tc_dq_buffers(const Problem &p, int bn, int stages)
{
    const int mode = mode_of(p.op);
    return dq_buffers(is_w4(mode) || mode == kW2A8, bn, stages, packed_group(p, bn, stages), kRowsW,
                      act_rows(bn, false));
}

// the deepest activation ring (2..5; 8 for token tiles up to 128, 16 up to 64) that keeps the grouped
// packed copies when K allows them
int tc_max_stages(const Problem &p, int bn)
{
    const int mode = mode_of(p.op);
    // grouped packed copies first (measured faster than one more activation stage without)
    const bool groupable = packed_group(p, bn, 2) == 4;
    for (int pg : {4, 1}) {
        if (pg == 4 && !groupable) continue;
        for (int s : {16, 8, 5, 4, 3, 2}) {
            if ((s == 16 && bn > 64) || (s == 8 && bn > 128)) continue;
            if (smem_bytes(mode, bn, s, pg) <= kMaxSmem) return s;
        }
    }
    return 2;
}

cudaError_t launch_tc(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream)
{
    if (!c.swap_ab) {
        if (p.op != QG_OP_W4A16) return cudaErrorInvalidValue;
        return p.interleaved ? launch_toka<kW4A16I>(p, c, err, stream)
                             : launch_toka<kW4A16>(p, c, err, stream);
    }
    switch (mode_of(p.op)) {
    case kDense: return launch_bn<kDense>(p, c, err, stream);
    case kW8A8: return launch_bn<kW8A8>(p, c, err, stream);
    case kW4A16:
        return p.interleaved ? launch_bn<kW4A16I>(p, c, err, stream)
                             : launch_bn<kW4A16>(p, c, err, stream);
    default:
        return p.interleaved ? launch_bn<kW2A8I>(p, c, err, stream)
                             : launch_bn<kW2A8>(p, c, err, stream);
    }
}

} // namespace qg
