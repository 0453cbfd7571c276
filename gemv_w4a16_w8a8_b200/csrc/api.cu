// C-ABI entry points of the qgemm library: argument checks, configuration choice (pinned
// table, then heuristic), the split-K output zeroing, the kernel launch and the error word.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "common.cuh"

// Device error word: kernels with bounded waits set it instead of trapping.
__device__ unsigned int g_qgemm_error_word;

namespace qg {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kDefaultSms = 148;   // B200
constexpr int kMaxSplit = 64;

std::mutex g_mu;

struct DeviceInfo {
    bool probed = false;
    bool sm100 = false;
    int sms = kDefaultSms;
    unsigned int *err_word = nullptr;
};
DeviceInfo g_dev[kMaxDevices];

using Key = std::tuple<int, int, int, int, int, int>;   // op, M, N, K, gs, has_zero
std::map<Key, qgemm_config_t> g_pinned;
bool g_cache_loaded = false;

// ------------------------------------------------------------------------------------------
qg_status probe_device(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return QG_ERR_CUDA;
        }
        d.sm100 = major == 10 && minor == 0;
        d.sms = sms > 0 ? sms : kDefaultSms;
        if (d.sm100) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_qgemm_error_word) != cudaSuccess) {
                cudaGetLastError();
                return QG_ERR_CUDA;
            }
            d.err_word = static_cast<unsigned int *>(p);
        }
        d.probed = true;
    }
    *out = &d;
    return d.sm100 ? QG_OK : QG_ERR_NOT_SM100;
}

int sm_count_or_default()
{
    int n = 0, dev = 0, sms = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || n <= 0 || cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return kDefaultSms;
    }
    return sms > 0 ? sms : kDefaultSms;
}

int effective_gs(int op, int K, int group_size)
{
    if (op != QG_OP_W4A16 && op != QG_OP_W4A16_INTERLEAVED) return K;
    return group_size <= 0 ? K : group_size;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape / flag rules shared by the matmul entry points, the planner and the tuner.
qg_status check_shape(int op, int M, int N, int K, int group_size, int has_zero, int split_k)
{
    if (op < QG_OP_W4A16 || op > QG_OP_W2A8_INTERLEAVED) return QG_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
    if (split_k > kMaxSplit) return QG_ERR_INVALID_ARG;
    if (has_zero != 0 && has_zero != 1) return QG_ERR_INVALID_ARG;
    switch (op) {
    case QG_OP_W4A16:
    case QG_OP_W4A16_INTERLEAVED: {
        if (K % 32) return QG_ERR_UNSUPPORTED_SHAPE;
        if (group_size < -1) return QG_ERR_INVALID_ARG;
        const int gs = effective_gs(op, K, group_size);
        if (gs % 32 || K % gs) return QG_ERR_UNSUPPORTED_SHAPE;
        break;
    }
    case QG_OP_W8A8:
    case QG_OP_W2A8:
    case QG_OP_W2A8_INTERLEAVED:
        if (group_size != -1 && group_size != 0) return QG_ERR_INVALID_ARG;
        if (has_zero) return QG_ERR_INVALID_ARG;
        if (K % (op == QG_OP_W8A8 ? 16 : 64)) return QG_ERR_UNSUPPORTED_SHAPE;
        break;
    case QG_OP_DENSE_F16:
        if (has_zero) return QG_ERR_INVALID_ARG;
        if (K % 8) return QG_ERR_UNSUPPORTED_SHAPE;
        break;
    }
    return QG_OK;
}

Problem make_problem(int op, const void *A, const void *W, const void *scales,
                     const void *zeros, void *C, int M, int N, int K, int group_size,
                     int has_zero)
{
    Problem p;
    p.op = op == QG_OP_W4A16_INTERLEAVED ? QG_OP_W4A16
                                         : (op == QG_OP_W2A8_INTERLEAVED ? QG_OP_W2A8 : op);
    p.interleaved = (op == QG_OP_W4A16_INTERLEAVED || op == QG_OP_W2A8_INTERLEAVED) ? 1 : 0;
    p.A = A;
    p.W = W;
    p.scales = scales;
    p.zeros = zeros;
    p.C = C;
    p.M = M;
    p.N = N;
    p.K = K;
    p.gs = effective_gs(op, K, group_size);
    p.has_zero = has_zero;
    return p;
}

size_t out_bytes(const Problem &p)
{
    const size_t elt = (p.op == QG_OP_W4A16 || p.op == QG_OP_DENSE_F16) ? 2 : 4;
    return (size_t)p.M * p.N * elt;
}

bool supports(const Problem &p, const qgemm_config_t &c)
{
    switch (c.path) {
    case QG_PATH_GEMV:
        if (p.op == QG_OP_W4A16) {
            if (c.bn == 2) return gemv_w4a16_h2_supports(p, c);
            return c.stages ? gemv_w4a16_tma_supports(p, c) : gemv_w4a16_supports(p, c);
        }
        if (p.op == QG_OP_W2A8 && c.stages) return gemv_w2a8_tma_supports(p, c);
        if (p.op == QG_OP_W8A8 || p.op == QG_OP_W2A8) return gemv_int_supports(p, c);
        return false;
    case QG_PATH_TC:
        return tc_supports(p, c);
    case QG_PATH_STREAM:
        return gemv_w4a16_stream_supports(p, c);
    default:
        return false;
    }
}

// ---- heuristic -------------------------------------------------------------------------------

int pick_split(long tiles, long work_units, long min_units_per_split, int sms)
{
    int split = 1;
    while (split < kMaxSplit && tiles * split < 4L * sms &&
           work_units / (2L * split) >= min_units_per_split)
        split *= 2;
    return split;
}

int pow2_at_least(int x, int lo, int hi)
{
    int v = lo;
    while (v < x && v < hi) v *= 2;
    return v;
}

int k_per_slab(int op) { return (op == QG_OP_DENSE_F16 || op == QG_OP_W4A16) ? 64 : 128; }

// tensor-core tile for M tokens: the token tile covers M (up to 256); the pipeline is as deep as
// shared memory allows (at most 4); K is split until the tiles fill every SM once.
qgemm_config_t tc_default(const Problem &p, int sms)
{
    qgemm_config_t c;
    std::memset(&c, 0, sizeof(c));
    c.path = QG_PATH_TC;
    c.bm = 128;
    c.bn = pow2_at_least(p.M, 16, 256);
    c.bk = k_per_slab(p.op);
    c.swap_ab = 1;
    // packed weights: the deepest ring that still leaves three dequant buffers (four for token
    // tiles of 128 and more, which hand them over slab by slab; both measured faster than a
    // deeper activation ring with fewer); other ops: the deepest ring that fits
    c.stages = tc_max_stages(p, c.bn);
    if (p.op == QG_OP_W4A16 || p.op == QG_OP_W2A8) {
        const int want = c.bn >= 128 ? 4 : 3;
        for (int st : {16, 8, 5, 4, 3, 2}) {
            if (st > c.stages) continue;
            qgemm_config_t t = c;
            t.stages = st;
            t.split_k = 1;
            c.stages = st;
            if (st == 2 || (tc_supports(p, t) && tc_dq_buffers(p, c.bn, st) >= want)) break;
        }
    }
    c.swap_ab = 1;
    const long tiles = (long)((p.N + 127) / 128) * ((p.M + c.bn - 1) / c.bn);
    const long nkb = (p.K + c.bk - 1) / c.bk;
    c.split_k = 1;
    while (c.split_k < 16 && tiles * c.split_k < sms && nkb / (2L * c.split_k) >= 4)
        c.split_k *= 2;
    return c;
}

// Token-major tensor-core tile for few tokens (W4A16): 128 tokens x 256 weight rows per tile, the
// deepest activation ring that keeps three upcast buffers, and the K split that gives the
// shortest persistent schedule: whole waves of units, each a run of 4-slab copies, plus a cost
// per unit for its epilogue, which grows with the tokens it adds into C (fp16 atomics).
qgemm_config_t tc_toka_default(const Problem &p, int sms)
{
    qgemm_config_t c;
    std::memset(&c, 0, sizeof(c));
    c.path = QG_PATH_TC;
    c.bm = 128;
    c.bn = 256;
    c.bk = 64;
    c.swap_ab = 0;
    c.split_k = 1;
    for (int st : {4, 3, 2}) {
        c.stages = st;
        if (tc_supports(p, c)) break;
    }
    const long tiles = (long)((p.N + 255) / 256) * ((p.M + 127) / 128);
    const int nkb = p.K / 64;
    double best = 1e30;
    for (int sk = 1; sk <= 16; ++sk) {
        const int kbps = ((nkb + sk - 1) / sk + 3) / 4 * 4;
        const int parts = (nkb + kbps - 1) / kbps;
        if (parts != sk) continue;   // another split gives the same parts
        const long units = tiles * parts;
        const double epi = 2.0 + (parts > 1 ? std::min(p.M, 128) / 8.0 : 0.0);
        const double cost = (double)((units + sms - 1) / sms) * (kbps + epi);
        if (cost < best) {
            best = cost;
            c.split_k = sk;
        }
    }
    return c;
}

// Persistent stream-K W4A16 kernel: 64-row x 512-K stages (256 contiguous bytes of each weight
// row a copy) consumed by 4 row warps x 2 K warps, in the deepest ring shared memory holds (up
// to 16 stages: HBM needs ~100 KB in flight per SM), one CTA per SM.
qgemm_config_t stream_default(const Problem &p)
{
    qgemm_config_t c;
    std::memset(&c, 0, sizeof(c));
    c.path = QG_PATH_STREAM;
    c.rows = 16;
    c.bm = 4;
    c.bn = 2;
    c.split_k = 1;
    for (int bk : {512, 256})
        for (int st = 16; st >= 2; --st) {
            c.bk = bk;
            c.stages = st;
            if (gemv_w4a16_stream_supports(p, c)) return c;
        }
    return c;
}

qgemm_config_t heuristic(const Problem &p, int sms, bool allow_stream)
{
    qgemm_config_t c;
    std::memset(&c, 0, sizeof(c));
    c.split_k = 1;
    // the persistent kernel wins from 9 tokens on (its shared operand table and atomics cost
    // more than they save below that; both are bound by the warp-level MMA rate)
    if (allow_stream && p.op == QG_OP_W4A16 && p.M > 8 && p.M <= 16) {
        qgemm_config_t st = stream_default(p);
        if (gemv_w4a16_stream_supports(p, st)) return st;
    }
    // token-major tensor-core tiles up to one tile of tokens (W4A16; groups of whole slabs)
    if (p.op == QG_OP_W4A16 && p.M > 16 && p.M <= 128) {
        qgemm_config_t tk = tc_toka_default(p, sms);
        if (tc_supports(p, tk)) return tk;
    }
    // tensor-core GEMM once there are enough tokens to fill its tile
    if (p.op == QG_OP_DENSE_F16 || p.M > 16) {
        qgemm_config_t tc = tc_default(p, sms);
        if (p.op == QG_OP_W4A16 && p.M >= 512) {
            // 512-token tiles (int4 weights): each upcast slab feeds two accumulators, which
            // measured a unit of 512 tokens at 1.71 units of 256 (1.17x the throughput); take
            // them when the persistent schedule of whole waves is shorter
            qgemm_config_t d = tc;
            d.bn = 512;
            d.stages = 4;
            d.split_k = 1;
            const long n_t = (p.N + 127) / 128;
            const long w256 = (n_t * ((p.M + 255) / 256) + sms - 1) / sms;
            const long w512 = (n_t * ((p.M + 511) / 512) + sms - 1) / sms;
            if (tc.bn == 256 && tc.split_k == 1 && 171 * w512 < 100 * w256 && tc_supports(p, d))
                return d;
        }
        if (tc_supports(p, tc)) return tc;
    }
    c.path = QG_PATH_GEMV;
    if (p.op == QG_OP_W4A16 && p.M == 1 && p.gs % 128 == 0 && p.K % 128 == 0) {
        // one token: the packed fp16 FMA-pipe GEMV (64-row tiles, 2-stage rings so that many
        // CTAs fit per SM), K split until the tiles fill the SMs about six times over while every
        // warp keeps at least four k-blocks
        c.rows = 64;
        c.bn = 2;
        c.stages = 2;
        const long tiles = (p.N + 63) / 64;
        const long nkb = p.K / 128;
        c.split_k = 1;
        while (c.split_k < 16 && tiles * c.split_k < 6L * sms && nkb / (2L * c.split_k) >= 4)
            c.split_k *= 2;
        return c;
    }
    if (p.op == QG_OP_W4A16) {
        c.rows = 32;
        const int kb = (p.gs % 128 == 0) ? 128 : (p.gs % 64 == 0 ? 64 : 32);
        const long tiles = (long)((p.N + 31) / 32) * ((p.M + 15) / 16);
        c.split_k = pick_split(tiles, p.K / kb, 12, sms);
        if (p.gs % 128 == 0) c.stages = 4;       // TMA-fed kernel
    } else if (p.op == QG_OP_W2A8 && p.K % 256 == 0) {
        c.rows = 64;                               // TMA-fed tensor-core kernel
        c.stages = 4;
        const long tiles = (long)((p.N + 63) / 64) * ((p.M + 15) / 16);
        c.split_k = pick_split(tiles, p.K / 256, 12, sms);
    } else {
        c.rows = 4;
        const int kc = p.op == QG_OP_W2A8 ? 64 : 16;
        const long tiles = (long)((p.N + 15) / 16) * ((p.M + 3) / 4);
        c.split_k = pick_split(tiles, p.K / kc, 128, sms);
    }
    return c;
}

// ---- pinned configurations ------------------------------------------------------------------------

bool parse_line(const char *line, Key *k, qgemm_config_t *c)
{
    int op, M, N, K, gs, hz;
    int v[8];
    if (std::sscanf(line, "%d %d %d %d %d %d %d %d %d %d %d %d %d %d", &op, &M, &N, &K, &gs, &hz,
                    &v[0], &v[1], &v[2], &v[3], &v[4], &v[5], &v[6], &v[7]) != 14)
        return false;
    *k = Key(op, M, N, K, gs, hz);
    c->path = v[0];
    c->rows = v[1];
    c->bm = v[2];
    c->bn = v[3];
    c->bk = v[4];
    c->stages = v[5];
    c->split_k = v[6];
    c->swap_ab = v[7];
    return true;
}

qg_status load_file_locked(const char *path)
{
    FILE *f = std::fopen(path, "r");
    if (!f) return QG_ERR_INVALID_ARG;
    char line[512];
    while (std::fgets(line, sizeof line, f)) {
        if (line[0] == '#') continue;
        Key k;
        qgemm_config_t c;
        if (!parse_line(line, &k, &c)) continue;
        Problem p = make_problem(std::get<0>(k), nullptr, nullptr, nullptr, nullptr, nullptr,
                                 std::get<1>(k), std::get<2>(k), std::get<3>(k), std::get<4>(k),
                                 std::get<5>(k));
        if (check_shape(std::get<0>(k), std::get<1>(k), std::get<2>(k), std::get<3>(k),
                        std::get<4>(k), std::get<5>(k), c.split_k) == QG_OK &&
            c.split_k >= 1 && supports(p, c))
            g_pinned[k] = c;   // entries that cannot run are skipped
    }
    std::fclose(f);
    return QG_OK;
}

void ensure_cache_loaded_locked()
{
    if (g_cache_loaded) return;
    g_cache_loaded = true;
    const char *path = std::getenv("QGEMM_CONFIG_CACHE");
    if (path && *path) load_file_locked(path);
}

Key key_of(const Problem &p)
{
    const int op = !p.interleaved ? p.op
                                  : (p.op == QG_OP_W2A8 ? (int)QG_OP_W2A8_INTERLEAVED
                                                        : (int)QG_OP_W4A16_INTERLEAVED);
    return Key(op, p.M, p.N, p.K, p.gs, p.has_zero);
}

qgemm_config_t choose(const Problem &p, int split_k, int sms)
{
    qgemm_config_t c;
    bool found = false;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        ensure_cache_loaded_locked();
        auto it = g_pinned.find(key_of(p));
        if (it != g_pinned.end()) {
            c = it->second;
            found = true;
        }
    }
    if (!found) c = heuristic(p, sms, split_k <= 0);
    if (split_k > 0) {
        // an explicit split asks for a path that cuts K into exactly that many parts
        if (c.path == QG_PATH_STREAM) c = heuristic(p, sms, false);
        if (c.path == QG_PATH_TC) c.rows = 0;   // not the stream-K schedule
        c.split_k = split_k;
    }
    return c;
}

// ---- dispatch ---------------------------------------------------------------------------------------

qg_status run(const Problem &p, const qgemm_config_t &c, DeviceInfo *d, cudaStream_t stream)
{
    if (!supports(p, c)) return QG_ERR_BAD_CONFIG;
    if (c.split_k > 1 || c.path == QG_PATH_STREAM || (c.path == QG_PATH_TC && c.rows == 1)) {
        if (cudaMemsetAsync(p.C, 0, out_bytes(p), stream) != cudaSuccess) {
            cudaGetLastError();
            return QG_ERR_CUDA;
        }
    }
    cudaError_t e = cudaErrorInvalidValue;
    if (c.path == QG_PATH_GEMV) {
        if (p.op == QG_OP_W4A16 && c.bn == 2)
            e = launch_gemv_w4a16_h2(p, c, d->err_word, stream);
        else if (p.op == QG_OP_W4A16)
            e = c.stages ? launch_gemv_w4a16_tma(p, c, d->err_word, stream)
                         : launch_gemv_w4a16(p, c, stream);
        else if (p.op == QG_OP_W2A8 && c.stages)
            e = launch_gemv_w2a8_tma(p, c, d->err_word, stream);
        else
            e = launch_gemv_int(p, c, stream);
    } else if (c.path == QG_PATH_TC) {
        e = launch_tc(p, c, d->err_word, stream);
    } else if (c.path == QG_PATH_STREAM) {
        Problem q = p;
        q.sms = d->sms;
        e = launch_gemv_w4a16_stream(q, c, d->err_word, stream);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status matmul(int op, const void *A, const void *W, const void *scales, const void *zeros,
                 void *C, int M, int N, int K, int group_size, int split_k, int has_zero,
                 cudaStream_t stream)
{
    qg_status s = check_shape(op, M, N, K, group_size, has_zero, split_k);
    if (s != QG_OK) return s;
    if (!A || !W || !C) return QG_ERR_INVALID_ARG;
    if (op == QG_OP_W4A16 || op == QG_OP_W4A16_INTERLEAVED) {
        if (!scales) return QG_ERR_INVALID_ARG;
        if ((zeros != nullptr) != (has_zero != 0)) return QG_ERR_INVALID_ARG;
        if (!aligned(scales, 2) || (zeros && !aligned(zeros, 2))) return QG_ERR_ALIGNMENT;
    }
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(C, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    Problem p = make_problem(op, A, W, scales, zeros, C, M, N, K, group_size, has_zero);
    return run(p, choose(p, split_k, d->sms), d, stream);
}

std::vector<qgemm_config_t> candidates(const Problem &p)
{
    std::vector<qgemm_config_t> out;
    qgemm_config_t c;
    std::memset(&c, 0, sizeof(c));
    if (p.op == QG_OP_W4A16 || p.op == QG_OP_W8A8 || p.op == QG_OP_W2A8) {
        c.path = QG_PATH_GEMV;
        const int rows16[] = {16, 32, 64};
        const int rows_int[] = {1, 2, 4, 8};
        const int rows_w2[] = {1, 2, 4, 8, 16, 32, 64};
        const int *rows = p.op == QG_OP_W4A16 ? rows16 : (p.op == QG_OP_W2A8 ? rows_w2 : rows_int);
        const int nrows = p.op == QG_OP_W4A16 ? 3 : (p.op == QG_OP_W2A8 ? 7 : 4);
        const int stage_opts[6] = {0, 2, 3, 4, 5, 6};  // 0: register-prefetch kernel
        for (int r = 0; r < nrows; ++r)
            for (int st = 0; st < (p.op == QG_OP_W8A8 ? 1 : 6); ++st)
                for (int s = 1; s <= 16; s *= 2) {
                    c.rows = rows[r];
                    c.stages = stage_opts[st];
                    c.split_k = s;
                    if (supports(p, c)) out.push_back(c);
                }
        if (p.op == QG_OP_W4A16 && p.M <= 8) {
            // 1..8 tokens on the packed fp16 FMA pipe (bn = 2)
            for (int rows : {32, 64})
                for (int st : {2, 3, 4, 5, 6})
                    for (int s = 1; s <= 16; s *= 2) {
                        c.rows = rows;
                        c.bn = 2;
                        c.stages = st;
                        c.split_k = s;
                        if (supports(p, c)) out.push_back(c);
                    }
            c.bn = 0;
        }
        if (p.op == QG_OP_W4A16 && p.M == 1) {
            // one token on the FMA pipe (TMA-fed kernel, bn = 1)
            for (int rows : {32, 64, 128})
                for (int st : {2, 3, 4, 5, 6})
                    for (int s = 1; s <= 16; s *= 2) {
                        c.rows = rows;
                        c.bn = 1;
                        c.stages = st;
                        c.split_k = s;
                        if (supports(p, c)) out.push_back(c);
                    }
            c.bn = 0;
        }
    }
    if (p.op == QG_OP_W4A16 && p.M <= 16) {
        // every stage shape and warp split, each at its deepest ring and at two-thirds of it
        qgemm_config_t t = stream_default(p);
        for (int bk : {256, 512, 1024})
            for (int wk : {1, 2, 4})
                for (int wr : {2, 3, 4, 6, 8}) {
                    t.bk = bk;
                    t.bn = wk;
                    t.bm = wr;
                    int deepest = 0;
                    for (int st = 2; st <= 16; ++st) {
                        t.stages = st;
                        if (supports(p, t)) deepest = st;
                    }
                    if (deepest == 0) continue;
                    t.stages = deepest;
                    out.push_back(t);
                    if (deepest * 2 / 3 >= 2 && deepest * 2 / 3 < deepest) {
                        t.stages = deepest * 2 / 3;
                        out.push_back(t);
                    }
                }
    }
    if (p.op == QG_OP_W4A16 && p.M <= 256) {
        qgemm_config_t t = tc_toka_default(p, kDefaultSms);
        const int best_split = t.split_k;
        for (int st : {2, 3, 4})
            for (int sk : {1, 2, 3, 4, 6, 8, 12, 16}) {
                t.stages = st;
                t.split_k = sk;
                if (tc_supports(p, t)) out.push_back(t);
            }
        t.split_k = best_split;
        for (int st : {2, 3, 4}) {
            t.stages = st;
            if (tc_supports(p, t)) out.push_back(t);
        }
    }
    if ((p.op == QG_OP_DENSE_F16 || p.op == QG_OP_W8A8) && p.M >= 256) {
        // the tile shared by a CTA pair (256 weight rows x 256 tokens): measured ahead of the
        // single-CTA tile for fp16 / int8 weights only (the packed formats lose on the
        // cross-SM hand-over of their upcast buffers)
        qgemm_config_t t = tc_default(p, kDefaultSms);
        t.bm = 256;
        t.bn = 256;
        for (int st : {4, 5})
            for (int sk : {1, 2}) {
                t.stages = st;
                t.split_k = sk;
                if (tc_supports(p, t)) out.push_back(t);
            }
    }
    if ((p.op == QG_OP_W4A16 || p.op == QG_OP_W2A8) && p.M >= 512) {
        // 512-token tile: each upcast weight slab feeds two 256-token accumulators
        qgemm_config_t t = tc_default(p, kDefaultSms);
        t.bn = 512;
        for (int st : {2, 4})
            for (int sk : {1, 2}) {
                t.stages = st;
                t.split_k = sk;
                const long tiles = (long)((p.N + 127) / 128) * ((p.M + 511) / 512);
                if (sk > 1 && tiles >= 2L * kDefaultSms) continue;
                if (tc_supports(p, t)) out.push_back(t);
            }
        // the same tile on the stream-K schedule
        t.stages = 4;
        t.split_k = 1;
        t.rows = 1;
        if (tc_supports(p, t)) out.push_back(t);
    }
    if (p.op != QG_OP_DENSE_F16 && p.M > 16) {
        // stream-K schedule of the default tensor-core tile (every SM an equal share of the work)
        qgemm_config_t t = (p.op == QG_OP_W4A16 && p.M <= 256) ? tc_toka_default(p, kDefaultSms)
                                                               : tc_default(p, kDefaultSms);
        t.split_k = 1;
        t.rows = 1;
        if (tc_supports(p, t)) out.push_back(t);
    }
    if (p.op == QG_OP_DENSE_F16 || p.M > 1) {
        const qgemm_config_t base = tc_default(p, kDefaultSms);
        const int bns[2] = {base.bn, base.bn / 2};
        for (int bi = 0; bi < 2; ++bi) {
            if (bns[bi] < 16) continue;
            for (int st : {2, 3, 4, 5, 8, 16})
                for (int sk = 1; sk <= 8; sk *= 2) {
                    qgemm_config_t t = base;
                    t.bn = bns[bi];
                    t.stages = st;
                    t.split_k = sk;
                    const long tiles = (long)((p.N + 127) / 128) * ((p.M + t.bn - 1) / t.bn);
                    if (sk > 1 && tiles >= 2L * kDefaultSms) continue;
                    if (tc_supports(p, t)) out.push_back(t);
                }
        }
    }
    return out;
}

} // namespace
} // namespace qg

using namespace qg;

namespace qg {
namespace {
struct HostPipe {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;                 // host-to-device, device-to-host
    cudaEvent_t start = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;   // one call's chain of records and waits at a time (events are reused)

bool pipe_init(HostPipe &hp)
{
    if (hp.ready) return true;
    const unsigned ev = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, ev) == cudaSuccess;
    for (int b = 0; b < 2 && ok; ++b)
        ok = cudaEventCreateWithFlags(&hp.in_done[b], ev) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.comp_done[b], ev) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.out_done[b], ev) == cudaSuccess;
    hp.ready = ok;
    return ok;
}

bool page_locked(const void *p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}
} // namespace
} // namespace qg

using namespace qg;

extern "C" {

qg_status qgemm_w4a16(const void *A, const uint32_t *Wq, const void *scales, const void *zeros,
                      void *C, int M, int N, int K, int group_size, int split_k, int has_zero,
                      cudaStream_t stream)
{
    return matmul(QG_OP_W4A16, A, Wq, scales, zeros, C, M, N, K, group_size, split_k, has_zero,
                  stream);
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// counters: one per output tile of the smallest row tile (16) and token tile (8) the streaming
// kernel uses, so the bound holds for every configuration; partials: split_k planes of M x N fp32
static size_t ws_counter_bytes(int M, int N)
{
    return align256((size_t)((N + 15) / 16) * (size_t)((M + 7) / 8) * sizeof(unsigned int));
}

size_t qgemm_w4a16_workspace_bytes(int M, int N, int K, int group_size, int split_k)
{
    if (check_shape(QG_OP_W4A16, M, N, K, group_size, 0, split_k) != QG_OK || split_k < 1)
        return 0;
    return ws_counter_bytes(M, N) + (size_t)split_k * M * N * sizeof(float);
}

qg_status qgemm_w4a16_splitk_f32(const void *A, const uint32_t *Wq, const void *scales,
                                 const void *zeros, void *C, int M, int N, int K, int group_size,
                                 int split_k, int has_zero, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream)
{
    qg_status s = check_shape(QG_OP_W4A16, M, N, K, group_size, has_zero, split_k);
    if (s != QG_OK) return s;
    if (split_k < 1) return QG_ERR_INVALID_ARG;
    if (effective_gs(QG_OP_W4A16, K, group_size) % 128) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!A || !Wq || !C || !scales || !workspace) return QG_ERR_INVALID_ARG;
    if ((zeros != nullptr) != (has_zero != 0)) return QG_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(Wq, 16) || !aligned(C, 16) || !aligned(workspace, 256) ||
        !aligned(scales, 2) || (zeros && !aligned(zeros, 2)))
        return QG_ERR_ALIGNMENT;
    if (workspace_bytes < qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k))
        return QG_ERR_INVALID_ARG;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    Problem p = make_problem(QG_OP_W4A16, A, Wq, scales, zeros, C, M, N, K, group_size, has_zero);
    qgemm_config_t c = choose(p, split_k, d->sms);
    if (c.path != QG_PATH_GEMV || c.stages == 0 || c.bn == 2) {   // this form lives in the TMA-fed kernel
        std::memset(&c, 0, sizeof(c));
        c.path = QG_PATH_GEMV;
        c.rows = 32;
        c.stages = 4;
    }
    c.split_k = split_k;
    if (!gemv_w4a16_tma_supports(p, c)) return QG_ERR_BAD_CONFIG;
    unsigned int *counters = static_cast<unsigned int *>(workspace);
    float *parts = reinterpret_cast<float *>(static_cast<char *>(workspace) + ws_counter_bytes(M, N));
    if (cudaMemsetAsync(counters, 0, gemv_w4a16_ws_tiles(p, c) * sizeof(unsigned int), stream) !=
        cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    if (launch_gemv_w4a16_tma(p, c, d->err_word, stream, parts, counters) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

// ---- host-buffer form: chunks of tokens through double buffers, copies on their own streams --

size_t qgemm_w4a16_host_workspace_bytes(int M, int N, int K, int chunk_tokens)
{
    if (M <= 0 || N <= 0 || K <= 0 || chunk_tokens < 0) return 0;
    const size_t mc = chunk_tokens ? (size_t)std::min(chunk_tokens, M) : (size_t)std::min(M, 1024);
    const size_t a = (mc * K * 2 + 255) / 256 * 256, c = (mc * N * 2 + 255) / 256 * 256;
    return 2 * (a + c);
}


qg_status qgemm_w4a16_host(const void *A_host, const uint32_t *Wq, const void *scales,
                           const void *zeros, void *C_host, int M, int N, int K, int group_size,
                           int split_k, int has_zero, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream)
{
    qg_status s = check_shape(QG_OP_W4A16, M, N, K, group_size, has_zero, split_k);
    if (s != QG_OK) return s;
    if (!A_host || !C_host || !Wq || !scales || !workspace) return QG_ERR_INVALID_ARG;
    if ((zeros != nullptr) != (has_zero != 0)) return QG_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(Wq, 16) || !aligned(scales, 2) ||
        (zeros && !aligned(zeros, 2)))
        return QG_ERR_ALIGNMENT;
    // chunk: the largest multiple of 256 tokens (or all M) whose double buffers fit
    const size_t per_token = 4 * ((size_t)K + (size_t)N);
    long mc = (long)std::min<size_t>((size_t)M, workspace_bytes / per_token);
    if (mc < M && mc >= 256) mc = mc / 256 * 256;   // whole 256-token tiles when there is room
    while (mc > 0 && qgemm_w4a16_host_workspace_bytes(M, N, K, (int)mc) > workspace_bytes)
        mc = mc > 256 ? mc - 256 : mc - 1;
    if (mc <= 0) return QG_ERR_INVALID_ARG;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    if (!page_locked(A_host) || !page_locked(C_host)) return QG_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    const size_t a_bytes = ((size_t)mc * K * 2 + 255) / 256 * 256;
    const size_t c_bytes = ((size_t)mc * N * 2 + 255) / 256 * 256;
    char *ws = static_cast<char *>(workspace);
    void *Ad[2] = {ws, ws + a_bytes};
    void *Cd[2] = {ws + 2 * a_bytes, ws + 2 * a_bytes + c_bytes};
    const char *Ah = static_cast<const char *>(A_host);
    char *Ch = static_cast<char *>(C_host);

    std::lock_guard<std::mutex> lk(g_pipe_mu);
    HostPipe &hp = g_pipe[dev];
    if (!pipe_init(hp)) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    bool good = ok(cudaEventRecord(hp.start, stream)) && ok(cudaStreamWaitEvent(hp.in, hp.start, 0)) &&
                ok(cudaStreamWaitEvent(hp.out, hp.start, 0));
    // chunks: a quarter-size first and last chunk when there are more than two (the first
    // copy in and the last copy out overlap nothing), full chunks between them
    std::vector<std::pair<long, long>> sched;   // (first token, tokens)
    {
        const long q = std::max(256L, mc / 4 / 256 * 256);
        const bool ramp = M > 2 * mc && q < mc;
        const long tail = ramp ? q : 0;
        long r = 0;
        if (ramp) {
            sched.push_back({0, q});
            r = q;
        }
        while (r < M - tail) {
            const long n = std::min(mc, M - tail - r);
            sched.push_back({r, n});
            r += n;
        }
        if (tail) sched.push_back({r, M - r});
    }
    const int chunks = (int)sched.size();
    for (int c = 0; c < chunks && good; ++c) {
        const int b = c & 1;
        const int rows = (int)sched[c].second;
        const size_t r0 = (size_t)sched[c].first;
        // A buffer b is free once the matmul of chunk c - 2 has finished reading it
        if (c >= 2) good = ok(cudaStreamWaitEvent(hp.in, hp.comp_done[b], 0));
        good = good && ok(cudaMemcpyAsync(Ad[b], Ah + r0 * K * 2, (size_t)rows * K * 2,
                                          cudaMemcpyHostToDevice, hp.in)) &&
               ok(cudaEventRecord(hp.in_done[b], hp.in)) &&
               ok(cudaStreamWaitEvent(stream, hp.in_done[b], 0));
        // C buffer b is free once the copy-out of chunk c - 2 has finished
        if (good && c >= 2) good = ok(cudaStreamWaitEvent(stream, hp.out_done[b], 0));
        if (!good) break;
        s = matmul(QG_OP_W4A16, Ad[b], Wq, scales, zeros, Cd[b], rows, N, K, group_size, split_k,
                   has_zero, stream);
        if (s != QG_OK) return s;
        good = ok(cudaEventRecord(hp.comp_done[b], stream)) &&
               ok(cudaStreamWaitEvent(hp.out, hp.comp_done[b], 0)) &&
               ok(cudaMemcpyAsync(Ch + r0 * N * 2, Cd[b], (size_t)rows * N * 2,
                                  cudaMemcpyDeviceToHost, hp.out)) &&
               ok(cudaEventRecord(hp.out_done[b], hp.out));
    }
    // work queued on `stream` later waits for every copy into C_host
    for (int b = 0; b < std::min(chunks, 2) && good; ++b)
        good = ok(cudaStreamWaitEvent(stream, hp.out_done[b], 0));
    if (!good) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status qgemm_w4a16_interleaved(const void *A, const uint32_t *Wq, const void *scales,
                                  const void *zeros, void *C, int M, int N, int K, int group_size,
                                  int split_k, int has_zero, cudaStream_t stream)
{
    return matmul(QG_OP_W4A16_INTERLEAVED, A, Wq, scales, zeros, C, M, N, K, group_size, split_k,
                  has_zero, stream);
}

qg_status quant_pack_int4_interleaved(const uint8_t *codes, uint32_t *packed, int M, int N, int K,
                                      int group_size, int split_k, int has_zero,
                                      cudaStream_t stream)
{
    (void)M; (void)group_size; (void)split_k; (void)has_zero;
    if (!codes || !packed || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
    if (K % 32) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(codes, 16) || !aligned(packed, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_pack_int4_interleaved(codes, packed, N, K, stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

// ---- qgemm_w4a16_splitk_f32_noalloc --------------------------------------------------------------
// For callers that must not allocate: the deterministic split-K scratch (arrival counters and
// fp32 partial tiles) lives in this fixed device buffer instead of a caller workspace. Every
// device that loads the library holds it until exit; all calls on a device share it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QGEMM_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};   // device address of g_noalloc_scratch, per device
}

qg_status qgemm_w4a16_splitk_f32_noalloc(const void *A, const uint32_t *Wq, const void *scales,
                                         const void *zeros, void *C, int M, int N, int K,
                                         int group_size, int split_k, int has_zero,
                                         cudaStream_t stream)
{
    qg_status s = check_shape(QG_OP_W4A16, M, N, K, group_size, has_zero, split_k);
    if (s != QG_OK) return s;
    if (split_k < 1) return QG_ERR_INVALID_ARG;
    if (effective_gs(QG_OP_W4A16, K, group_size) % 128) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!A || !Wq || !C || !scales) return QG_ERR_INVALID_ARG;
    if ((zeros != nullptr) != (has_zero != 0)) return QG_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(Wq, 16) || !aligned(C, 16) || !aligned(scales, 2) ||
        (zeros && !aligned(zeros, 2)))
        return QG_ERR_ALIGNMENT;
    const size_t need = qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k);
    if (need == 0) return QG_ERR_INVALID_ARG;
    if (need > (size_t)QGEMM_NOALLOC_SCRATCH_BYTES) return QG_ERR_SCRATCH_TOO_SMALL;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    void *scratch = nullptr;
    {
        // once per device, with that device current: the buffer's device address (in host
        // code the symbol itself is only a stand-in and must never reach a kernel)
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void *ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
                cudaGetLastError();
                return QG_ERR_CUDA;
            }
            g_noalloc_ptr[dev] = ptr;
        }
        scratch = g_noalloc_ptr[dev];
    }
    Problem p = make_problem(QG_OP_W4A16, A, Wq, scales, zeros, C, M, N, K, group_size, has_zero);
    qgemm_config_t c = choose(p, split_k, d->sms);
    if (c.path != QG_PATH_GEMV || c.stages == 0 || c.bn == 2) {
        std::memset(&c, 0, sizeof(c));
        c.path = QG_PATH_GEMV;
        c.rows = 32;
        c.stages = 4;
    }
    c.split_k = split_k;
    if (!gemv_w4a16_tma_supports(p, c)) return QG_ERR_BAD_CONFIG;
    unsigned int *counters = static_cast<unsigned int *>(scratch);
    float *parts = reinterpret_cast<float *>(static_cast<char *>(scratch) + ws_counter_bytes(M, N));
    // the arrival counters must start at zero; the partial tiles are overwritten in full
    if (cudaMemsetAsync(counters, 0, gemv_w4a16_ws_tiles(p, c) * sizeof(unsigned int), stream) !=
        cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    if (launch_gemv_w4a16_tma(p, c, d->err_word, stream, parts, counters) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status qgemm_w8a8(const int8_t *A, const int8_t *W, int32_t *C, int M, int N, int K,
                     int group_size, int split_k, int has_zero, cudaStream_t stream)
{
    return matmul(QG_OP_W8A8, A, W, nullptr, nullptr, C, M, N, K, group_size, split_k, has_zero,
                  stream);
}

qg_status qgemm_w8a8_requant(const int8_t *A, const int8_t *W, const float *mult, int8_t *C,
                             int M, int N, int K, cudaStream_t stream)
{
    qg_status s = check_shape(QG_OP_W8A8, M, N, K, -1, 0, 1);
    if (s != QG_OK) return s;
    if (!A || !W || !mult || !C) return QG_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(mult, 4)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    Problem p = make_problem(QG_OP_W8A8, A, W, nullptr, nullptr, C, M, N, K, -1, 0);
    p.mult = mult;
    // rounding needs the whole sum: one K part, never atomics
    qgemm_config_t c = choose(p, 1, d->sms);
    if (c.split_k != 1 || !supports(p, c)) return QG_ERR_BAD_CONFIG;
    return run(p, c, d, stream);
}

qg_status qgemm_w2a8(const int8_t *A, const uint32_t *Wq, int32_t *C, int M, int N, int K,
                     int group_size, int split_k, int has_zero, cudaStream_t stream)
{
    return matmul(QG_OP_W2A8, A, Wq, nullptr, nullptr, C, M, N, K, group_size, split_k, has_zero,
                  stream);
}

qg_status qgemm_w2a8_interleaved(const int8_t *A, const uint32_t *Wq, int32_t *C, int M, int N,
                                 int K, int group_size, int split_k, int has_zero,
                                 cudaStream_t stream)
{
    return matmul(QG_OP_W2A8_INTERLEAVED, A, Wq, nullptr, nullptr, C, M, N, K, group_size, split_k,
                  has_zero, stream);
}

qg_status qgemm_dense_f16(const void *A, const void *W, void *C, int M, int N, int K,
                          int split_k, cudaStream_t stream)
{
    return matmul(QG_OP_DENSE_F16, A, W, nullptr, nullptr, C, M, N, K, -1, split_k, 0, stream);
}

qg_status quant_pack_int4(const uint8_t *codes, uint32_t *packed, int M, int N, int K,
                          int group_size, int split_k, int has_zero, cudaStream_t stream)
{
    (void)M; (void)group_size; (void)split_k; (void)has_zero;
    if (!codes || !packed || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
    if (K % 32) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(codes, 16) || !aligned(packed, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_pack_int4(codes, packed, N, K, stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status quant_rtn_int4(const void *W, uint32_t *Wq, void *scales, void *zeros, int N, int K,
                         int group_size, int has_zero, cudaStream_t stream)
{
    if (!W || !Wq || !scales || N <= 0 || K <= 0 || group_size < -1) return QG_ERR_INVALID_ARG;
    if (has_zero != 1 || !zeros) return QG_ERR_INVALID_ARG;   // unsigned codes need the zero point
    if (K % 32) return QG_ERR_UNSUPPORTED_SHAPE;
    const int gs = group_size <= 0 ? K : group_size;
    if (K % gs || !(gs == 32 || gs == 64 || gs == 128 || gs % 256 == 0))
        return QG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(scales, 2) || !aligned(zeros, 2))
        return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_rtn_int4(static_cast<const __half *>(W), Wq, static_cast<__half *>(scales),
                        static_cast<__half *>(zeros), N, K, gs, stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status quant_pack_int2(const int8_t *vals, uint32_t *packed, int M, int N, int K,
                          int group_size, int split_k, int has_zero, cudaStream_t stream)
{
    (void)M; (void)group_size; (void)split_k; (void)has_zero;
    if (!vals || !packed || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
    if (K % 64) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(vals, 16) || !aligned(packed, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_pack_int2(vals, packed, N, K, stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status quant_pack_int2_interleaved(const int8_t *vals, uint32_t *packed, int M, int N, int K,
                                      int group_size, int split_k, int has_zero,
                                      cudaStream_t stream)
{
    (void)M; (void)group_size; (void)split_k; (void)has_zero;
    if (!vals || !packed || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
    if (K % 64) return QG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(vals, 16) || !aligned(packed, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_pack_int2_interleaved(vals, packed, N, K, stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status qgemm_plan(int op, int M, int N, int K, int group_size, int has_zero, int split_k,
                     qgemm_config_t *out)
{
    if (!out) return QG_ERR_INVALID_ARG;
    qg_status s = check_shape(op, M, N, K, group_size, has_zero, split_k);
    if (s != QG_OK) return s;
    Problem p = make_problem(op, nullptr, nullptr, nullptr, nullptr, nullptr, M, N, K, group_size,
                             has_zero);
    *out = choose(p, split_k, sm_count_or_default());
    return supports(p, *out) ? QG_OK : QG_ERR_BAD_CONFIG;
}

qg_status qgemm_set_config(int op, int M, int N, int K, int group_size, int has_zero,
                           const qgemm_config_t *cfg)
{
    qg_status s = check_shape(op, M, N, K, group_size, has_zero, cfg ? cfg->split_k : 0);
    if (s != QG_OK) return s;
    Problem p = make_problem(op, nullptr, nullptr, nullptr, nullptr, nullptr, M, N, K, group_size,
                             has_zero);
    std::lock_guard<std::mutex> lk(g_mu);
    ensure_cache_loaded_locked();
    if (!cfg) {
        g_pinned.erase(key_of(p));
        return QG_OK;
    }
    if (cfg->split_k < 1 || !supports(p, *cfg)) return QG_ERR_BAD_CONFIG;
    g_pinned[key_of(p)] = *cfg;
    return QG_OK;
}

qg_status qgemm_tune(int op, const void *A, const void *W, const void *scales,
                     const void *zeros, void *C, int M, int N, int K, int group_size,
                     int has_zero, int reps, cudaStream_t stream, qgemm_config_t *best)
{
    qg_status s = check_shape(op, M, N, K, group_size, has_zero, 0);
    if (s != QG_OK) return s;
    const bool w4 = op == QG_OP_W4A16 || op == QG_OP_W4A16_INTERLEAVED;
    if (!A || !W || !C || (w4 && !scales)) return QG_ERR_INVALID_ARG;
    if (w4 && (zeros != nullptr) != (has_zero != 0)) return QG_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(C, 16)) return QG_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    s = probe_device(&d);
    if (s != QG_OK) return s;
    if (reps <= 0) reps = 20;
    Problem p = make_problem(op, A, W, scales, zeros, C, M, N, K, group_size, has_zero);
    std::vector<qgemm_config_t> cands = candidates(p);
    if (cands.empty()) return QG_ERR_BAD_CONFIG;
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    // A timeout raised by work queued before the search belongs to that work's caller: report
    // it now instead of charging it to a candidate (or losing it when the word is cleared).
    unsigned int word = 0;
    const unsigned int zero = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess ||
        cudaMemcpyFromSymbol(&word, g_qgemm_error_word, sizeof(word)) != cudaSuccess) {
        cudaGetLastError();
        cudaEventDestroy(e0);
        cudaEventDestroy(e1);
        return QG_ERR_CUDA;
    }
    if (word) {
        cudaEventDestroy(e0);
        cudaEventDestroy(e1);
        return QG_ERR_DEVICE_TIMEOUT;
    }
    float best_ms = 1e30f;
    bool have_winner = false;
    qgemm_config_t winner = cands[0];
    qg_status result = QG_OK;
    for (const qgemm_config_t &c : cands) {
        for (int i = 0; i < 2 && result == QG_OK; ++i) result = run(p, c, d, stream);
        if (result != QG_OK) break;
        if (cudaEventRecord(e0, stream) != cudaSuccess) result = QG_ERR_CUDA;
        for (int i = 0; i < reps && result == QG_OK; ++i) result = run(p, c, d, stream);
        if (result == QG_OK && cudaEventRecord(e1, stream) != cudaSuccess) result = QG_ERR_CUDA;
        if (result != QG_OK || cudaEventSynchronize(e1) != cudaSuccess) {
            if (result == QG_OK) result = QG_ERR_CUDA;
            break;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess) {
            result = QG_ERR_CUDA;
            break;
        }
        // a candidate whose kernels gave up a bounded wait is dropped, and the word cleared so
        // that the next candidate (and later callers) start clean
        if (cudaMemcpyFromSymbol(&word, g_qgemm_error_word, sizeof(word)) != cudaSuccess) {
            result = QG_ERR_CUDA;
            break;
        }
        if (word) {
            if (cudaMemcpyToSymbol(g_qgemm_error_word, &zero, sizeof(zero)) != cudaSuccess) {
                result = QG_ERR_CUDA;
                break;
            }
            continue;
        }
        if (ms < best_ms) {
            best_ms = ms;
            winner = c;
            have_winner = true;
        }
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaGetLastError();
    if (result != QG_OK) return result;
    if (!have_winner) return QG_ERR_DEVICE_TIMEOUT;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        ensure_cache_loaded_locked();
        g_pinned[key_of(p)] = winner;
    }
    if (best) *best = winner;
    return QG_OK;
}

qg_status qgemm_save_configs(const char *path)
{
    if (!path) return QG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    FILE *f = std::fopen(path, "w");
    if (!f) return QG_ERR_INVALID_ARG;
    std::fprintf(f, "# op M N K group_size has_zero path rows bm bn bk stages split_k swap_ab\n");
    for (const auto &kv : g_pinned) {
        const Key &k = kv.first;
        const qgemm_config_t &c = kv.second;
        std::fprintf(f, "%d %d %d %d %d %d %d %d %d %d %d %d %d %d\n", std::get<0>(k),
                     std::get<1>(k), std::get<2>(k), std::get<3>(k), std::get<4>(k),
                     std::get<5>(k), c.path, c.rows, c.bm, c.bn, c.bk, c.stages, c.split_k,
                     c.swap_ab);
    }
    std::fclose(f);
    return QG_OK;
}

qg_status qgemm_load_configs(const char *path)
{
    if (!path) return QG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_cache_loaded = true;
    return load_file_locked(path);
}

void qgemm_clear_configs(void)
{
    std::lock_guard<std::mutex> lk(g_mu);
    g_cache_loaded = true;
    g_pinned.clear();
}

qg_status qgemm_selftest_bounded_wait(int limit_us, cudaStream_t stream)
{
    if (limit_us < 1 || limit_us > 2000000) return QG_ERR_INVALID_ARG;
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (launch_wait_selftest(d->err_word, 1000ull * (unsigned long long)limit_us, stream) !=
        cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

qg_status qgemm_sync_check(cudaStream_t stream)
{
    DeviceInfo *d = nullptr;
    qg_status s = probe_device(&d);
    if (s != QG_OK) return s;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    unsigned int word = 0;
    const unsigned int zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_qgemm_error_word, sizeof(word)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_qgemm_error_word, &zero, sizeof(zero)) != cudaSuccess) {
        cudaGetLastError();
        return QG_ERR_CUDA;
    }
    return word ? QG_ERR_DEVICE_TIMEOUT : QG_OK;
}

const char *qgemm_status_string(qg_status status)
{
    switch (status) {
    case QG_OK: return "ok";
    case QG_ERR_INVALID_ARG: return "invalid argument";
    case QG_ERR_ALIGNMENT: return "pointer not aligned as required";
    case QG_ERR_UNSUPPORTED_SHAPE: return "unsupported K / group_size";
    case QG_ERR_CUDA: return "CUDA runtime or launch error";
    case QG_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case QG_ERR_NOT_SM100: return "device is not compute capability 10.0 (B200)";
    case QG_ERR_BAD_CONFIG: return "configuration cannot run this problem";
    case QG_ERR_SCRATCH_TOO_SMALL:
        return "problem needs more scratch than the library's fixed buffer holds";
    }
    return "unknown status";
}

int qgemm_version(void) { return 100; }

} // extern "C"
