// W4A16 small-M persistent streaming kernel ("stream-K" GEMV), path QG_PATH_STREAM.
//
// At M <= 16 the matmul is bound by HBM: every packed weight is read once and the arithmetic
// per byte is small, so the kernel is built to keep the copy engine busy and the issue slots
// free for the weight arithmetic:
//   * The work is split evenly over a persistent grid. The (row block, K stage) units of the
//     whole problem are laid out row block by row block and every CTA takes one contiguous run
//     of them, so no SM idles in a partial last wave and the pipeline never drains between
//     tiles. A row block whose K range two CTAs share meets in C through red.global.add
//     (parallel-k with atomic reduction, hidet-org/hidet issue #364), so C is zeroed first.
//   * One producer warp moves each unit into a ring of shared-memory stages with TMA: the
//     weights of all the CTA's rows as a 3-D box of 128-byte chunks under the 128-byte swizzle,
//     256 or 512 contiguous bytes of every row (long runs keep HBM efficient), and the
//     activations of the stage's K range. It then turns the activations into the MMA operand
//     pairs and the per-group correction sums once for the whole CTA. Multi-stage pipelining
//     with a searchable depth is the same issue's topic.
//   * The consumer warps only upcast weights and run the MMAs. Warp (wr, wk) owns 16 rows and
//     every WK-th 128-K sub-block of each stage, so a stage is shared by WR x WK warps; at the
//     end of a row block the WK partial sums meet in shared memory and leave as one f16x2
//     atomic per row pair and token. The arithmetic per 16 x 128 block is the warp-level
//     scheme of w4a16_frag.cuh, with scale and zero applied per group in fp32.
#include <algorithm>
#include <mutex>

#include "sm100.cuh"
#include "w4a16_frag.cuh"

namespace qg {
namespace {

constexpr int kSub = 128;          // K values per sub-block (one fragment pass)
constexpr int kMaxConsumers = 15;  // consumer warps a CTA may have (plus the copy warp: 16 warps)
constexpr int kMaxStages = 16;

// Slot row that holds MMA fragment row g (0..7). One 128-bit shared load of a warp is served in
// four phases of eight lanes, i.e. fragment rows 2q and 2q + 1; their 16-byte pieces fall in
// opposite halves of the 128-byte bank window when the swizzle patterns of their lines differ in
// bit 2. The line of row r, chunk c is r * CH + c, so the rows are permuted to make that so.
template <int CH> __device__ __forceinline__ int slot_row(int g)
{
    if constexpr (CH == 4) return g;
    else if constexpr (CH == 2) return ((g >> 1) & 1) | ((g & 1) << 1) | (g & 4);
    else return (g >> 1) | ((g & 1) << 2);
}

// Shared-memory plan of one CTA (bytes; the ring's parts start on 1024-byte boundaries). With
// `tab`, the operand pairs and correction sums of the whole K range are prepared once into a
// table and the ring holds weights only; otherwise every stage carries its activations and its
// prepared operands.
struct StreamPlan {
    int rows;        // weight rows per unit (16 per row warp)
    int w_slot;      // packed weights of one stage
    int a_slot;      // activations of one stage, M x stage K fp16 (0 with the table)
    int p_slot;      // prepared operands of one stage (0 with the table)
    int red;         // partial sums of every consumer warp (16 rows x 8 NT tokens fp32)
    int table;       // prepared operands of every sub-block of K (0 without the table)
    int stages;
    __host__ __device__ static int up1k(int x) { return (x + 1023) & ~1023; }
    // operand pairs of one sub-block: [word j][token][lane t] uint4, tokens < M only; then per
    // token tile and lane t the float4 (corr 2t, corr 2t+1, sum a 2t, sum a 2t+1)
    __host__ __device__ static int pair_bytes(int M) { return 4 * M * 4 * 16; }
    __host__ __device__ static int sub_bytes(int M, int nt) { return pair_bytes(M) + nt * 4 * 16; }
    __host__ __device__ StreamPlan(int row_warps, int k_warps, int ch, int nt, int M, int st, int K,
                                   bool tab)
    {
        rows = 16 * row_warps;
        w_slot = rows * ch * 128;
        a_slot = tab ? 0 : up1k(M * 256 * ch * 2);
        p_slot = tab ? 0 : up1k(2 * ch * sub_bytes(M, nt));
        red = row_warps * k_warps * 16 * 8 * nt * 4;
        table = tab ? up1k((K / 128) * sub_bytes(M, nt)) : 0;
        stages = st;
    }
    __host__ __device__ int stage_bytes() const { return w_slot + a_slot + p_slot; }
    __host__ __device__ int table_offset() const { return stages * stage_bytes(); }
    __host__ __device__ int red_offset() const { return table_offset() + table; }
    __host__ __device__ int bar_offset() const { return red_offset() + red; }
    // 1 KB alignment slack, the ring, the table, the partial sums, three barriers a stage, the
    // consumers' rendezvous barrier and an abort flag
    __host__ __device__ size_t total() const
    {
        return 1024 + (size_t)bar_offset() + (size_t)24 * stages + 8 + 16;
    }
};

// The operands one task produces: token tile t of one 128-K sub-block. `act(j)` gives this lane's
// 8 activations j (token 8 t + g, K values 32 t' + 8 j of the sub-block; zero past M); the pairs
// go to pp, the correction sums (lanes 0..3) to pc.
template <typename ActFn>
__device__ __forceinline__ void make_operands(ActFn act, bool ilv, int M, int t, int lg, int lt,
                                              uint4 *pp, float4 *pc)
{
    const int tok = 8 * t + lg;
    uint32_t corr_op[4];
    w4_corr_operand(corr_op);
    uint32_t b[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 v = act(j);
        if (ilv) w4_act_pairs<true>(v, b[j]);
        else w4_act_pairs<false>(v, b[j]);
        if (tok < M) pp[(j * M + tok) * 4 + lt] = make_uint4(b[j][0], b[j][1], b[j][2], b[j][3]);
    }
    // corr (rows 0..7) and sum a (rows 8..15), four short chains
    float q[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int e = 0; e < 4; ++e) q[x][e] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        mma_16816_f16(q[(j & 1) * 2], corr_op, b[j][0], b[j][1], q[(j & 1) * 2]);
        mma_16816_f16(q[(j & 1) * 2 + 1], corr_op, b[j][2], b[j][3], q[(j & 1) * 2 + 1]);
    }
    // every row of the constant operand is the same: lanes 0..3 hold the sums
    if (lg == 0) {
        float cz[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) cz[e] = (q[0][e] + q[1][e]) + (q[2][e] + q[3][e]);
        pc[t * 4 + lt] = make_float4(cz[0], cz[1], cz[2], cz[3]);
    }
}

// CH: 128-byte weight chunks (256 K values) per row and stage. NT: 8-token MMA tiles
// (M <= 8 * NT). WK: consumer warps that share a row block, each taking every WK-th sub-block
// of a stage. TAB: the operands of the whole K range are prepared once into a table (else every
// stage brings its activations and the consumers prepare them, one task per warp). Block:
// WR * WK consumer warps, then the copy warp.
template <int CH, int NT, int WK, bool TAB>
__global__ void __launch_bounds__((kMaxConsumers + 1) * 32, 1)
gemv_w4a16_stream_kernel(const __grid_constant__ CUtensorMap tm_w,
                         const __grid_constant__ CUtensorMap tm_a, const __half *__restrict__ A,
                         const __half *__restrict__ S, const __half *__restrict__ Z,
                         __half *__restrict__ C, int M, int N, int K, int gs, int stages, int ilv,
                         unsigned int *err)
{
    constexpr int kStageK = 256 * CH, kSubs = 2 * CH, kPer = kSubs / WK;
    static_assert(kSubs % WK == 0, "sub-blocks split evenly over the K warps");
    const int W = (int)(blockDim.x >> 5) - 1;   // consumer warps; warp W issues the copies
    const int WR = W / WK;
    const StreamPlan plan(WR, WK, CH, NT, M, stages, K, TAB);
    extern __shared__ uint8_t dsmem_raw[];
    uint8_t *dsmem = dsmem_raw + ((1024u - (smem_u32(dsmem_raw) & 1023u)) & 1023u);
    float *red = reinterpret_cast<float *>(dsmem + plan.red_offset());
    uint64_t *full = reinterpret_cast<uint64_t *>(dsmem + plan.bar_offset());
    uint64_t *pfull = full + stages;
    uint64_t *empty = pfull + stages;
    uint64_t *meet = empty + stages;                  // consumers' rendezvous
    int &abort_flag = *reinterpret_cast<int *>(meet + 1);
    const int stage_bytes = plan.stage_bytes();
    auto w_slot = [&](int s) { return dsmem + (size_t)s * stage_bytes; };
    auto a_slot = [&](int s) { return dsmem + (size_t)s * stage_bytes + plan.w_slot; };
    // prepared operands of sub-block sub of the unit in stage s (or, with the table, of the
    // sub-block at index sub of K)
    const int sub_bytes = StreamPlan::sub_bytes(M, NT);
    auto p_base = [&](int s, int sub) -> uint8_t * {
        if constexpr (TAB) return dsmem + plan.table_offset() + (size_t)sub * sub_bytes;
        else return dsmem + (size_t)s * stage_bytes + plan.w_slot + plan.a_slot + (size_t)sub * sub_bytes;
    };
    auto p_pairs = [&](int s, int sub) { return reinterpret_cast<uint4 *>(p_base(s, sub)); };
    auto p_corr = [&](int s, int sub) {
        return reinterpret_cast<float4 *>(p_base(s, sub) + StreamPlan::pair_bytes(M));
    };

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int lg = lane >> 2, lt = lane & 3;
    const int nst = (K + kStageK - 1) / kStageK;
    const long long total = (long long)((N + plan.rows - 1) / plan.rows) * nst;
    const long long u0 = total * blockIdx.x / gridDim.x;
    const int cnt = (int)(total * (blockIdx.x + 1) / gridDim.x - u0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&pfull[s]), W);
            mbar_init(smem_u32(&empty[s]), W);
        }
        mbar_init(smem_u32(meet), W);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async_smem();
    }
    __syncthreads();
    volatile int *abort_v = &abort_flag;
    // unit cursor (super-block of plan.rows rows, K stage), advanced without divisions
    const int sb0 = (int)(u0 / nst), st0 = (int)(u0 % nst);
    const uint32_t tx_bytes = (uint32_t)(plan.w_slot + (TAB ? 0 : M * kStageK * 2));

    if (warp == W) {
        // ---------------- copy warp: keeps every free stage of the ring in flight ----------------
        if (lane == 0) {
            int j_sb = sb0, j_st = st0, slot = 0;
            uint32_t lap = 0;   // (j / stages) & 1
            int j = 0;
            for (; j < cnt; ++j) {
                // the stage's previous unit, j - stages, must be consumed: its release is the
                // completion of the empty barrier's phase number j / stages - 1
                if (j >= stages) {
                    if (!mbar_wait(smem_u32(&empty[slot]), lap ^ 1u, abort_v, err)) break;
                }
                const uint32_t bar = smem_u32(&full[slot]);
                mbar_expect_tx(bar, tx_bytes);
                tma_load_3d(smem_u32(w_slot(slot)), &tm_w, bar, 0, j_st * CH, j_sb * plan.rows);
                if constexpr (!TAB)
                    tma_load_3d(smem_u32(a_slot(slot)), &tm_a, bar, 0, j_st * 4 * CH, 0);
                if (++j_st == nst) {
                    j_st = 0;
                    ++j_sb;
                }
                if (++slot == stages) {
                    slot = 0;
                    lap ^= 1u;
                }
            }
            // Copies of the last `stages` units may still be in flight when a wait gave up; every
            // earlier one was consumed. Let them land before the CTA exits (bounded).
            int dummy = 0;
            for (int u = max(0, j - stages); u < j; ++u)
                mbar_wait(smem_u32(&full[u % stages]), (uint32_t)((u / stages) & 1), &dummy, nullptr);
        }
        return;
    }
    // ------------- consumers: warp (wr, wk) = (warp % WR, warp / WR) -------------------------
    const int wr = warp % WR, wk = warp / WR;
    const int G = K / gs;
    const bool zero_pt = Z != nullptr;
    // fragment row g lives in unit row 16 wr + rho(g) (rows g + 8 eight further); the 128-byte
    // line of its chunk c is that row * CH + c, and 16 wr CH lines keep the swizzle pattern
    const int rho = slot_row<CH>(lg);
    const int wrow = 16 * wr + rho;
    const int base_line = wrow * CH;

    // all consumer warps meet (bounded: a warp that gave up a wait never arrives)
    uint32_t meet_phase = 0;
    auto rendezvous = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(meet));
        const bool ok = mbar_wait(smem_u32(meet), meet_phase, abort_v, err);
        meet_phase ^= 1u;
        return __all_sync(0xffffffffu, ok);
    };
    float acc[NT][4];
    auto zero_acc = [&]() {
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
    };
    zero_acc();
    // Partial sums of super-block sb: the WK warps of each row block meet in shared memory, then
    // the sums leave for C (zeroed by the caller) as one atomic per row pair and token.
    auto flush = [&](int sb) -> bool {
        float *mine = red + (size_t)warp * 8 * NT * 16;   // [token][16 rows]
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                mine[(8 * t + 2 * lt + (e & 1)) * 16 + rho + 8 * (e >> 1)] = acc[t][e];
        if (!rendezvous()) return false;
        const int pairs = plan.rows / 2;
        const bool even_n = (N & 1) == 0;
        for (int idx = threadIdx.x; idx < pairs * M; idx += 32 * W) {
            const int tok = idx / pairs, row = 2 * (idx - tok * pairs);
            const int rw = row >> 4, r16 = row & 15;
            float v0 = 0.f, v1 = 0.f;
#pragma unroll
            for (int k = 0; k < WK; ++k) {
                const float *p = red + ((size_t)(k * WR + rw) * 8 * NT + tok) * 16 + r16;
                v0 += p[0];
                v1 += p[1];
            }
            const int grow = sb * plan.rows + row;
            __half *dst = C + (size_t)tok * N + grow;
            if (grow + 1 < N && even_n) {
                red_add_f16x2(dst, pack_half2_rn(v0, v1));
            } else {
                if (grow < N) red_add_f16(dst, half_bits_rn(v0));
                if (grow + 1 < N) red_add_f16(dst + 1, half_bits_rn(v1));
            }
        }
        return rendezvous();   // the partial sums are read before the next flush writes them
    };
    // scale / zero bits of this warp's sub-blocks of the next unit, loaded one unit ahead
    uint16_t sn[kPer][2], zn[kPer][2];
    auto load_scales = [&](int sb, int st) {
        const int rbase = sb * plan.rows + wrow;
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int g = min((st * kStageK + kSub * (wk + WK * m)) / gs, G - 1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const size_t gi = (size_t)min(rbase + 8 * h, N - 1) * G + g;
                sn[m][h] = ld_cached_u16(S + gi);
                zn[m][h] = zero_pt ? ld_cached_u16(Z + gi) : (uint16_t)0;
            }
        }
    };
    // Operand preparation. With the table: task k = (sub-block k / NT of K, token tile k % NT)
    // belongs to consumer warp k % W, once, before any unit. Without: the same split over the
    // sub-blocks of each unit; every warp prepares its share of the next unit before it
    // consumes the current one, then waits for all shares (pfull, count W).
    auto prep = [&](int ps, int pst) {
        const int nsub = min(kSubs, (K - pst * kStageK) / kSub);
        const uint8_t *as = a_slot(ps);
        for (int k = warp; k < nsub * NT; k += W) {
            const int sub = k / NT, t = k - sub * NT;
            const int tok = 8 * t + lg;
            auto act = [&](int j) {
                return tok < M ? *reinterpret_cast<const uint4 *>(
                                     as + ((size_t)tok * kStageK + kSub * sub + 32 * lt + 8 * j) * 2)
                               : make_uint4(0u, 0u, 0u, 0u);
            };
            make_operands(act, ilv != 0, M, t, lg, lt, p_pairs(ps, sub), p_corr(ps, sub));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&pfull[ps]));
    };

    int c_sb = sb0, c_st = st0;
    if (cnt > 0) load_scales(c_sb, c_st);
    int cur_sb = -1, consumed = 0, s = 0;
    uint32_t phase = 0;
    bool ok = true;
    if constexpr (TAB) {
        const int ntask = (K / kSub) * NT;
        for (int k = warp; k < ntask; k += W) {
            const int sub = k / NT, t = k - sub * NT;
            const int tok = 8 * t + lg;
            const __half *arow = A + (size_t)min(tok, M - 1) * K + kSub * sub + 32 * lt;
            auto act = [&](int j) {
                return tok < M ? ld_cached_v4(arow + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
            };
            make_operands(act, ilv != 0, M, t, lg, lt, p_pairs(0, sub), p_corr(0, sub));
        }
        ok = rendezvous();
    } else if (cnt > 0) {
        ok = mbar_wait(smem_u32(&full[0]), 0u, abort_v, err);
        if (ok) prep(0, st0);
    }
    for (int i = 0; ok && i < cnt; ++i) {
        const int sb = c_sb, st = c_st;
        if (++c_st == nst) {   // the unit after this one
            c_st = 0;
            ++c_sb;
        }
        if constexpr (!TAB) {
            // this warp's share of the next unit's operands
            if (i + 1 < cnt) {
                const int ns = s + 1 == stages ? 0 : s + 1;
                const uint32_t nph = s + 1 == stages ? phase ^ 1u : phase;
                if (!mbar_wait(smem_u32(&full[ns]), nph, abort_v, err)) break;
                prep(ns, c_st);
            }
        }
        const int nsub = min(kSubs, (K - st * kStageK) / kSub);
        if (sb != cur_sb) {
            if (cur_sb >= 0 && !flush(cur_sb)) break;
            zero_acc();
            cur_sb = sb;
        }
        float sc[kPer][2], zr[kPer][2];
#pragma unroll
        for (int m = 0; m < kPer; ++m)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sc[m][h] = half_bits_to_float(sn[m][h]);
                zr[m][h] = half_bits_to_float(zn[m][h]);
            }
        if (i + 1 < cnt) load_scales(c_sb, c_st);
        if constexpr (TAB) {
            if (!mbar_wait(smem_u32(&full[s]), phase, abort_v, err)) break;
        } else {
            // every warp waited for this unit's copy before preparing its share; all shares are in
            if (!mbar_wait(smem_u32(&pfull[s]), phase, abort_v, err)) break;
        }
        const uint8_t *ws = w_slot(s);
        const int sub0 = TAB ? st * kSubs : 0;   // index of the unit's first sub-block operands
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int sub = wk + WK * m;
            if (sub >= nsub) break;
            uint32_t b[NT][4][4];
            float cz[NT][4];
            const uint4 *pp = p_pairs(s, sub0 + sub);
            const float4 *pc = p_corr(s, sub0 + sub);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int tok = 8 * t + lg;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = tok < M ? pp[(j * M + tok) * 4 + lt] : make_uint4(0u, 0u, 0u, 0u);
                    b[t][j][0] = v.x;
                    b[t][j][1] = v.y;
                    b[t][j][2] = v.z;
                    b[t][j][3] = v.w;
                }
                const float4 q = pc[t * 4 + lt];
                cz[t][0] = q.x;
                cz[t][1] = q.y;
                cz[t][2] = q.z;
                cz[t][3] = q.w;
            }
            // this lane's 16-byte piece: chunk sub / 2, pieces 4..7 for odd sub-blocks
            const int line = base_line + (sub >> 1);
            const uint32_t off = (uint32_t)(line * 128 + 16 * ((lt ^ (line & 7)) ^ (4 * (sub & 1))));
            const uint4 wa = *reinterpret_cast<const uint4 *>(ws + off);
            const uint4 wb = *reinterpret_cast<const uint4 *>(ws + off + 8 * CH * 128);
            const uint32_t wva[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wvb[4] = {wb.x, wb.y, wb.z, wb.w};
            float d[NT][4][4];   // four accumulation chains of two MMAs each
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[t][x][e] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    w4_word_mma(wva[j], wvb[j], b[t][j], d[t][(j & 1) * 2], d[t][(j & 1) * 2 + 1]);
            // d: (row g, tok 2t) (row g, tok 2t+1) (row g+8, tok 2t) (row g+8, tok 2t+1)
            // cz: corr of tok 2t, 2t+1, then sum a of tok 2t, 2t+1
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = e >> 1, tk = e & 1;
                    const float dd = (d[t][0][e] + d[t][1][e]) + (d[t][2][e] + d[t][3][e]);
                    acc[t][e] += sc[m][h] * (dd - cz[t][tk] - zr[m][h] * cz[t][2 + tk]);
                }
        }
        consumed = i + 1;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        if (++s == stages) {
            s = 0;
            phase ^= 1u;
        }
    }
    if (cur_sb >= 0 && consumed == cnt) flush(cur_sb);
}


template <int CH, int NT, int WK, bool TAB>
cudaError_t launch_one(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                       cudaStream_t stream)
{
    auto kern = gemv_w4a16_stream_kernel<CH, NT, WK, TAB>;
    static std::mutex mu;
    static bool opted_in[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!opted_in[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 227 * 1024);
            if (e != cudaSuccess) return e;
            opted_in[dev] = true;
        }
    }
    const StreamPlan plan(c.bm, WK, CH, NT, p.M, c.stages, p.K, TAB);
    // W as 3-D: 32 words of a 128-byte chunk, K / 256 chunks, N rows (128-byte swizzle)
    const uint64_t wd[3] = {32, (uint64_t)p.K / 256, (uint64_t)p.N};
    const uint64_t ws[2] = {128, (uint64_t)p.K / 2};
    const uint32_t wb[3] = {32, (uint32_t)CH, (uint32_t)plan.rows};
    // A as 3-D: 64 halves of a 128-byte chunk, K / 64 chunks, M rows (all of them)
    const uint64_t ad[3] = {64, (uint64_t)p.K / 64, (uint64_t)p.M};
    const uint64_t as[2] = {128, (uint64_t)p.K * 2};
    const uint32_t ab[3] = {64, (uint32_t)(4 * CH), (uint32_t)p.M};
    CUtensorMap tw, ta;
    if (!make_map_3d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.W, wd, ws, wb,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT16, p.A, ad, as, ab,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const long long units = (long long)((p.N + plan.rows - 1) / plan.rows) *
                            ((p.K + 256 * CH - 1) / (256 * CH));
    const long long ctas = std::max(1LL, std::min((long long)p.sms, units));
    kern<<<(unsigned)ctas, (c.bm * WK + 1) * 32, plan.total(), stream>>>(
        tw, ta, static_cast<const __half *>(p.A), static_cast<const __half *>(p.scales),
        p.has_zero ? static_cast<const __half *>(p.zeros) : nullptr, static_cast<__half *>(p.C),
        p.M, p.N, p.K, p.gs, c.stages, p.interleaved, err);
    return cudaGetLastError();
}

// The operand table of the whole K range when it fits beside the configured ring.
bool use_table(const Problem &p, const qgemm_config_t &c)
{
    const StreamPlan t(c.bm, c.bn, c.bk / 256, p.M <= 8 ? 1 : 2, p.M, c.stages, p.K, true);
    return t.total() <= 227 * 1024;
}

template <int CH, int WK>
cudaError_t launch_nt(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream)
{
    const bool tab = use_table(p, c);
    if (p.M <= 8)
        return tab ? launch_one<CH, 1, WK, true>(p, c, err, stream)
                   : launch_one<CH, 1, WK, false>(p, c, err, stream);
    return tab ? launch_one<CH, 2, WK, true>(p, c, err, stream)
               : launch_one<CH, 2, WK, false>(p, c, err, stream);
}

template <int CH>
cudaError_t launch_wk(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                      cudaStream_t stream)
{
    if (c.bn == 1) return launch_nt<CH, 1>(p, c, err, stream);
    if (c.bn == 2) return launch_nt<CH, 2>(p, c, err, stream);
    if constexpr (CH >= 2) return launch_nt<CH, 4>(p, c, err, stream);
    return cudaErrorInvalidValue;
}

} // namespace

bool gemv_w4a16_stream_supports(const Problem &p, const qgemm_config_t &c)
{
    if (p.op != QG_OP_W4A16 || p.M < 1 || p.M > 16 || p.gs % kSub != 0 || p.K % 256 != 0)
        return false;
    if (c.rows != 16 || (c.bk != 256 && c.bk != 512 && c.bk != 1024)) return false;
    if (c.bn != 1 && c.bn != 2 && c.bn != 4) return false;
    if ((2 * c.bk / 256) % c.bn != 0) return false;                 // sub-blocks split evenly
    if (c.bm < 1 || c.bm * c.bn > kMaxConsumers || c.bm > 16) return false;   // box <= 256 rows
    if (c.stages < 2 || c.stages > kMaxStages) return false;
    if (use_table(p, c)) return true;
    const StreamPlan plan(c.bm, c.bn, c.bk / 256, p.M <= 8 ? 1 : 2, p.M, c.stages, p.K, false);
    return plan.total() <= 227 * 1024;
}

cudaError_t launch_gemv_w4a16_stream(const Problem &p, const qgemm_config_t &c, unsigned int *err,
                                     cudaStream_t stream)
{
    if (c.bk == 256) return launch_wk<1>(p, c, err, stream);
    if (c.bk == 512) return launch_wk<2>(p, c, err, stream);
    return launch_wk<4>(p, c, err, stream);
}

} // namespace qg
