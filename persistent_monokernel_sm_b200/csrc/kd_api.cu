// kd_api.cu -- host side of libkd: configuration checks, the arena layout, weight repacking
// into the streaming layout, and the C ABI declared in include/kd.h.
#include <cuda_runtime.h>
#include <algorithm>
#include <vector>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "kd.h"
#include "kd_layout.h"

using namespace kd;

namespace {

constexpr int kMaxGrid = 256;  // attention-record room for up to this many CTAs

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool valid_config(const kd_config* c) {
    if (!c) return false;
    if (c->n_layers < 1 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0) return false;
    if (c->head_dim != 64 && c->head_dim != 128) return false;
    if (c->n_heads % c->n_kv_heads || c->n_heads / c->n_kv_heads > kMaxGroup) return false;
    if (c->n_kv_heads > kMaxKvHeads) return false;
    Shape sh;
    if (!make_shape(c->d_model, &sh)) return false;
    if (c->ffn_dim <= 0 || c->vocab < 1 || c->max_seq < 1) return false;
    if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f)) return false;
    return true;
}

Dims make_dims(const kd_config* c) {
    Dims d;
    d.L = c->n_layers, d.d = c->d_model, d.Hq = c->n_heads, d.Hkv = c->n_kv_heads, d.hd = c->head_dim;
    d.F = c->ffn_dim, d.V = c->vocab, d.S = c->max_seq, d.eps = c->rms_eps, d.theta = c->rope_theta;
    d.qd = d.Hq * d.hd, d.kvd = d.Hkv * d.hd, d.r = d.Hq / d.Hkv;
    d.qkv_rows = d.qd + 2 * d.kvd;
    return d;
}

Layout make_layout(const Dims& d) {
    Layout y;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    const size_t D = d.d;
    y.embed = take((size_t)d.V * D * 2);
    y.lm_head = take((size_t)d.V * D * 2);
    y.final_norm = take(D * 2);
    y.layer0 = off;
    size_t lo = 0;
    auto ltake = [&](size_t bytes) {
        size_t at = lo;
        lo = align256(lo + bytes);
        return at;
    };
    y.l_attn_norm = ltake(D * 2);
    y.l_ffn_norm = ltake(D * 2);
    y.l_wqkv = ltake((size_t)d.qkv_rows * D * 2);
    y.l_wot = ltake((size_t)d.qd * D * 2);
    y.l_wgu = ltake((size_t)2 * d.F * D * 2);
    y.l_wdt = ltake((size_t)d.F * D * 2);
    y.layer_stride = lo;
    off = y.layer0 + (size_t)d.L * y.layer_stride;
    y.weights_end = off;
    y.rope = take((size_t)d.S * (d.hd / 2) * 8);  // RoPE table, filled by kd_load_weights
    const size_t kv = (size_t)d.L * d.Hkv * d.S * d.hd * 2;
    y.kcache = take(kv);
    y.vcache = take(kv);
    y.kv_bytes = 2 * kv;
    y.delta = take((size_t)3 * kSumCopies * D * 4);                // split-K sums, 3 rotating buffers
    y.qkv = take((size_t)d.qkv_rows * 8);                          // tagged q / k / v of the step
    y.rec = take((size_t)kMaxGrid * d.r * (d.hd + 2) * 8);         // tagged attention records
    y.ctl = take((size_t)kCtlWords * 8);
    y.syncw = take(sync_region_bytes());
    y.dietab = take(kMaxSmid);
    y.tokens_in = take((size_t)d.S * 4);
    y.tokens_out = take((size_t)d.S * 4);  // staging for kd_generate
    y.total = off;
    return y;
}

// End of the scratch that starts at zero and is cleared after a failed run: the split-K
// buffers, the tagged words, the control words and the sync counter replicas.
size_t scratch_end(const Layout& y) { return y.syncw + sync_region_bytes(); }

// Die probe, run once by kd_create: each CTA records its SM id and, for each of the ncand
// candidate counter words (kDieBlock bytes apart), the shortest round trip of a few atomics
// that add 0. Its outputs go to a scratch region of the arena that is cleared afterwards.
__global__ void die_probe(unsigned long long* cand, int ncand, int* smid_out, unsigned int* lat_out) {
    if (threadIdx.x != 0) return;
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    smid_out[blockIdx.x] = (int)sm;
    for (int j = 0; j < ncand; ++j) {
        unsigned long long* w = cand + (size_t)j * (kDieBlock / 8);
        long long best = 1LL << 62;
        for (int r = 0; r < 6; ++r) {
            const long long t0 = clock64();
            unsigned long long old, dep;
            asm volatile("atom.relaxed.gpu.global.add.u64 %0, [%1], 0;" : "=l"(old) : "l"(w) : "memory");
            asm volatile("shr.b64 %0, %1, 63;" : "=l"(dep) : "l"(old));  // the clock waits for the answer
            const long long dt = clock64() + (long long)dep - t0;
            if (r > 0 && dt < best) best = dt;
        }
        lat_out[blockIdx.x * ncand + j] = (unsigned int)(best > 0xffffffffLL ? 0xffffffffu : best);
    }
}

}  // namespace

struct kd_ctx {
    kd_config cfg;
    Dims dm;
    Layout lay;
    Shape sh;
    uint8_t* arena;
    cudaStream_t stream;
    int device;
    int nb, smem, ns, pieces, blk, work_floats, hin_floats;
    bool has_weights, failed;
    int pos, n_pending;
    long long launches;
    long long timeout_ns;
    float inv_temp;            // 0: greedy
    unsigned long long seed;   // sampling stream
    size_t sync_off[2];        // sync counter replicas (arena byte offsets)
    int nsync;
    uint32_t tag;  // tag base of the next launch (advanced by the tagged phases each launch runs)
    unsigned long long* trace;
    int trace_every, trace_rows;
    char err[512];
};

static int fail(kd_ctx* c, int code, const char* fmt, ...) {
    if (c) {
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(c->err, sizeof c->err, fmt, ap);
        va_end(ap);
    }
    return code;
}

#define KD_CUDA(ctx, call)                                                                       \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess)                                                                   \
            return fail((ctx), KD_ECUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
    } while (0)

// ------------------------------------------------------------------ repack kernels

namespace {

// Row r of the kv-head-major [q; k; v] projection of one layer. Kv head g owns rows
// [g * (r + 2) * hd, (g + 1) * (r + 2) * hd): its r q heads, its k head, its v head. q and k
// heads hold RoPE pairs (i, i + hd/2) in adjacent rows (2i, 2i + 1); v rows keep their order.
__global__ void repack_qkv(uint8_t* dst_layer0, size_t layer_stride, size_t off, const uint16_t* wq,
                           const uint16_t* wk, const uint16_t* wv, Dims dm) {
    const int row = blockIdx.x, l = blockIdx.y;
    const int per = (dm.r + 2) * dm.hd;
    const int g = row / per, rr = row % per;
    const int seg = rr / dm.hd, j = rr % dm.hd;
    const int pj = (j >> 1) + ((j & 1) ? dm.hd / 2 : 0);  // RoPE-pair order
    const uint16_t* src;
    if (seg < dm.r) src = wq + ((size_t)l * dm.qd + (size_t)(g * dm.r + seg) * dm.hd + pj) * dm.d;
    else if (seg == dm.r) src = wk + ((size_t)l * dm.kvd + (size_t)g * dm.hd + pj) * dm.d;
    else src = wv + ((size_t)l * dm.kvd + (size_t)g * dm.hd + j) * dm.d;
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst_layer0 + (size_t)l * layer_stride + off + (size_t)row * dm.d * 2);
    for (int i = threadIdx.x; i < dm.d / 8; i += blockDim.x) d[i] = s[i];
}

// dst rows (2i, 2i + 1) = (gate row i, up row i)
__global__ void repack_gu(uint8_t* dst_layer0, size_t layer_stride, size_t off, const uint16_t* wg,
                          const uint16_t* wu, Dims dm) {
    const int r = blockIdx.x, l = blockIdx.y;
    const uint16_t* src = ((r & 1) ? wu : wg) + ((size_t)l * dm.F + (r >> 1)) * dm.d;
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst_layer0 + (size_t)l * layer_stride + off + (size_t)r * dm.d * 2);
    for (int i = threadIdx.x; i < dm.d / 8; i += blockDim.x) d[i] = s[i];
}

// dst [cols][rows] = src [rows][cols]^T for every layer (bf16), 32 x 32 tiles. Used for the
// output projection ([d][Hq*hd] -> [Hq*hd][d]) and the down projection ([d][F] -> [F][d]),
// so that a CTA's split-K share of either is one contiguous run of rows.
__global__ void transpose_bf16(uint8_t* dst_layer0, size_t layer_stride, size_t off, const uint16_t* src, int rows,
                               int cols) {
    __shared__ uint16_t tile[32][33];
    const int l = blockIdx.z;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    const uint16_t* s = src + (size_t)l * rows * cols;
    uint16_t* d = reinterpret_cast<uint16_t*>(dst_layer0 + (size_t)l * layer_stride + off);
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = s[(size_t)r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < cols) d[(size_t)c * rows + r] = tile[threadIdx.x][i];
    }
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Shared-memory scratch (floats) of one CTA, sized for the largest user:
//  hin:  the CTA's hidden values (down-projection inputs) or attention output dims;
//  work: row-GEMV partials (rows x slices) of the Q/K/V, gate/up and LM-head shares, the
//        attention scores and reductions of one softmax block, the split-K group sums, and
//        the attention records the output projection gathers.
void scratch_sizes(const Dims& d, const Shape& sh, int nb, int pieces, int blk, int* hin, int* work) {
    const int units = (d.F + nb - 1) / nb + 1;
    const int cols = d.r * d.hd / pieces + 2;
    *hin = ((units > cols ? units : cols) + 31) & ~31;
    const int gm = d.r <= 2 ? 2 : d.r <= 4 ? 4 : 8;
    long long w = 0;
    auto need = [&](long long v) { if (v > w) w = v; };
    const int pairs = (d.r + 2) * d.hd / 2;
    need((long long)2 * ((pairs + pieces - 1) / pieces) * sh.gs);  // Q/K/V rows
    need((long long)2 * units * sh.gs);                             // gate/up rows
    need((long long)((d.V + nb - 1) / nb) * sh.gs);                 // LM-head rows
    const int pps = kStageBytes / (2 * d.hd), nq = d.hd / 32, npg = kConsumerThreads / (d.hd / 2);
    const long long spart = 2LL * nq * gm * pps, vred = (long long)npg * gm * d.hd;
    need((long long)(blk + 1) * gm + (spart > vred ? spart : vred));  // attention
    if (sh.ug > 1) need((long long)sh.ug * d.d);                    // split-K group sums
    need((long long)pieces * (4 + cols));                           // gathered attention records
    *work = (int)((w + 31) & ~31LL);
}

}  // namespace

// ------------------------------------------------------------------ internal accessors

int kd_internal_view(kd_ctx* c, kd_ctx_view* v) {
    if (!c || !v) return KD_EINVAL;
    v->dm = &c->dm;
    v->lay = &c->lay;
    v->sh = &c->sh;
    v->arena = c->arena;
    v->stream = c->stream;
    v->device = c->device, v->nb = c->nb, v->smem = c->smem, v->ns = c->ns;
    v->pieces = c->pieces, v->blk = c->blk, v->work_floats = c->work_floats, v->hin_floats = c->hin_floats;
    v->timeout_ns = c->timeout_ns;
    v->has_weights = c->has_weights;
    v->inv_temp = c->inv_temp;
    v->seed = c->seed;
    v->sync_off[0] = c->sync_off[0], v->sync_off[1] = c->sync_off[1];
    v->nsync = c->nsync;
    return KD_OK;
}

int kd_internal_fail(kd_ctx* c, int code, const char* msg) { return fail(c, code, "%s", msg); }

void kd_internal_count_launch(kd_ctx* c) { c->launches += 1; }

namespace kd {
// The launch parameters that depend only on the handle (shared with kd_decode_noalloc).
void fill_launch_shape(const kd_ctx_view& v, Params& p) {
    p.dm = *v.dm;
    p.sh = *v.sh;
    p.nb = v.nb;
    p.ns = v.ns;
    p.pieces = v.pieces;
    p.blk = v.blk;
    p.work_floats = v.work_floats;
    p.hin_floats = v.hin_floats;
    p.timeout_ns = v.timeout_ns;
    p.inv_temp = v.inv_temp;
    p.seed_lo = (uint32_t)(v.seed & 0xffffffffull);
    p.seed_hi = (uint32_t)(v.seed >> 32);
    p.sync_off[0] = v.sync_off[0], p.sync_off[1] = v.sync_off[1];
    p.nsync = v.nsync;
}
}  // namespace kd

// ------------------------------------------------------------------ C ABI

extern "C" {

size_t kd_arena_bytes(const kd_config* cfg) {
    if (!valid_config(cfg)) return 0;
    return make_layout(make_dims(cfg)).total;
}

double kd_step_bytes(const kd_config* cfg, int64_t kv_positions, int with_head) {
    if (!valid_config(cfg) || kv_positions < 0) return -1.0;
    const double d = cfg->d_model, hd = cfg->head_dim, Hq = cfg->n_heads, Hkv = cfg->n_kv_heads;
    const double F = cfg->ffn_dim, L = cfg->n_layers, V = cfg->vocab;
    // per layer: two norm gains, Wq/Wk/Wv, Wo, gate/up, down
    const double layer = 2 * d + (Hq + 2 * Hkv) * hd * d + Hq * hd * d + 2 * F * d + F * d;
    double elems = L * layer + d;  // + the embedding row of the input token
    if (with_head) elems += d + V * d;
    const double kv = L * Hkv * (double)kv_positions * hd * 2;  // K and V rows
    return 2.0 * (elems + kv);
}

// Which die owns which counter word, and which replica is local to each SM. The candidates
// are kDieBlock-aligned words of the sync region; candidate 0 is replica 0; replica 1 is the
// first candidate whose round trips differ from candidate 0's by more than 1.4x for the
// median CTA (the two are then homed on different dies); each SM takes the replica with the
// shorter round trip. With no such candidate (one die, or a probe that saw no difference)
// there is one replica. Correctness never depends on the outcome: every CTA adds to every
// replica, and a wrong local choice only costs latency.
static int probe_dies(kd_ctx* c) {
    const uintptr_t a0 = (uintptr_t)(c->arena + c->lay.syncw);
    const uintptr_t al = (a0 + kDieBlock - 1) & ~(uintptr_t)(kDieBlock - 1);
    const size_t base = (size_t)(al - (uintptr_t)c->arena);
    c->sync_off[0] = c->sync_off[1] = base;
    c->nsync = 1;
    const int nb = c->nb, K = kDieCandidates;
    // outputs in the attention-record scratch (cleared below, before any decode)
    int* d_smid = reinterpret_cast<int*>(c->arena + c->lay.rec);
    unsigned int* d_lat = reinterpret_cast<unsigned int*>(c->arena + c->lay.rec + 4096);
    if ((size_t)4096 + (size_t)nb * K * 4 > (size_t)kMaxGrid * c->dm.r * (c->dm.hd + 2) * 8)
        return fail(c, KD_EINVAL, "die probe: scratch too small");
    die_probe<<<nb, 32, 0, c->stream>>>(reinterpret_cast<unsigned long long*>(c->arena + base), K, d_smid, d_lat);
    std::vector<int> smid(nb);
    std::vector<unsigned int> lat((size_t)nb * K);
    KD_CUDA(c, cudaGetLastError());
    KD_CUDA(c, cudaMemcpyAsync(smid.data(), d_smid, (size_t)nb * 4, cudaMemcpyDeviceToHost, c->stream));
    KD_CUDA(c, cudaMemcpyAsync(lat.data(), d_lat, (size_t)nb * K * 4, cudaMemcpyDeviceToHost, c->stream));
    KD_CUDA(c, cudaStreamSynchronize(c->stream));
    int r1 = -1;
    for (int j = 1; j < K && r1 < 0; ++j) {
        std::vector<double> ratio(nb);
        for (int b = 0; b < nb; ++b) {
            const double x = lat[(size_t)b * K], y = lat[(size_t)b * K + j];
            ratio[b] = (x > y ? x : y) / ((x < y ? x : y) > 1.0 ? (x < y ? x : y) : 1.0);
        }
        std::nth_element(ratio.begin(), ratio.begin() + nb / 2, ratio.end());
        if (ratio[nb / 2] > 1.4) r1 = j;
    }
    std::vector<uint8_t> tab(kMaxSmid, 0);
    if (r1 > 0) {
        for (int b = 0; b < nb; ++b)
            if (smid[b] >= 0 && smid[b] < kMaxSmid) tab[smid[b]] = lat[(size_t)b * K + r1] < lat[(size_t)b * K] ? 1 : 0;
        c->sync_off[1] = base + (size_t)r1 * kDieBlock;
        c->nsync = 2;
    }
    KD_CUDA(c, cudaMemcpyAsync(c->arena + c->lay.dietab, tab.data(), kMaxSmid, cudaMemcpyHostToDevice, c->stream));
    KD_CUDA(c, cudaMemsetAsync(c->arena + c->lay.delta, 0, scratch_end(c->lay) - c->lay.delta, c->stream));
    KD_CUDA(c, cudaStreamSynchronize(c->stream));
    return KD_OK;
}

int kd_create(const kd_config* cfg, void* d_arena, size_t arena_bytes, void* stream, kd_ctx** out) {
    if (!out) return KD_EINVAL;
    *out = nullptr;
    if (!valid_config(cfg) || !d_arena) return KD_EINVAL;
    kd_ctx* c = (kd_ctx*)calloc(1, sizeof(kd_ctx));
    if (!c) return KD_EINVAL;
    c->cfg = *cfg;
    c->dm = make_dims(cfg);
    c->lay = make_layout(c->dm);
    make_shape(c->dm.d, &c->sh);
    c->arena = (uint8_t*)d_arena;
    c->stream = (cudaStream_t)stream;
    c->timeout_ns = 1000000000LL;
    if (const char* t = getenv("KD_TIMEOUT_MS")) c->timeout_ns = atoll(t) * 1000000LL;
    int rc = KD_OK;
    if (arena_bytes < c->lay.total || ((uintptr_t)d_arena & 255)) {
        rc = fail(c, KD_ENOMEM, "arena of %zu bytes at %p; need %zu bytes, 256-byte aligned", arena_bytes,
                  d_arena, c->lay.total);
    }
    cudaDeviceProp prop;
    if (rc == KD_OK) {
        cudaError_t e = cudaGetDevice(&c->device);
        if (e == cudaSuccess) e = cudaGetDeviceProperties(&prop, c->device);
        if (e != cudaSuccess) rc = fail(c, KD_ECUDA, "device query failed: %s", cudaGetErrorString(e));
    }
    if (rc == KD_OK && !prop.cooperativeLaunch) rc = fail(c, KD_ECOOP, "device lacks cooperative launch");
    if (rc == KD_OK) {
        const Dims& d = c->dm;
        c->nb = prop.multiProcessorCount;
        if (c->nb > kMaxGrid) c->nb = kMaxGrid;
        c->pieces = c->nb / d.Hkv;
        if (c->pieces < 1) rc = fail(c, KD_EINVAL, "%d CTAs cannot serve %d kv heads", c->nb, d.Hkv);
    }
    if (rc == KD_OK) {
        // The ring takes what the scratch leaves: the largest softmax block (a multiple of a
        // stage's positions, at most 1024) that still leaves room for 4 stages, then as many
        // stages as fit (at most kMaxStages).
        const Dims& d = c->dm;
        const int pps = kStageBytes / (2 * d.hd);
        Params p{};
        p.dm = d;
        c->ns = 0;
        for (int blk = 1024; blk >= pps && c->ns == 0; blk -= pps) {
            scratch_sizes(d, c->sh, c->nb, c->pieces, blk, &c->hin_floats, &c->work_floats);
            p.hin_floats = c->hin_floats;
            p.work_floats = c->work_floats;
            p.ns = 0;
            const int fixed = monokernel_smem_bytes(p);
            const int ns = (kSmemLimit - fixed) / kStageBytes;
            if (ns >= 4) {
                c->ns = ns > kMaxStages ? kMaxStages : ns;
                c->blk = blk;
            }
        }
        if (c->ns == 0) rc = fail(c, KD_EINVAL, "shared-memory scratch leaves no room for a pipeline");
        if (rc == KD_OK) {
            p.ns = c->ns;
            c->smem = monokernel_smem_bytes(p);
            int per_sm = 0;
            int e = monokernel_occupancy(d, c->smem, &per_sm);
            if (e != 0) rc = fail(c, KD_ECUDA, "occupancy query failed: %s", cudaGetErrorString((cudaError_t)e));
            else if (per_sm < 1)
                rc = fail(c, KD_ECOOP, "monokernel cannot be resident (smem %d bytes)", c->smem);
        }
    }
    if (rc == KD_OK) {
        // Control words, the split-K buffers and the tagged words start at zero: tag 0 is
        // never expected (the first launch's phases carry tags 1, 2, ...).
        cudaError_t e = cudaMemsetAsync(c->arena + c->lay.delta, 0, scratch_end(c->lay) - c->lay.delta,
                                        c->stream);
        if (e != cudaSuccess) rc = fail(c, KD_ECUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    }
    if (rc == KD_OK) rc = probe_dies(c);
    if (rc != KD_OK) {
        fprintf(stderr, "kd_create: %s\n", c->err);
        free(c);
        return rc;
    }
    *out = c;
    return KD_OK;
}

int kd_load_weights(kd_ctx* c, const kd_weights* w) {
    if (!c || !w) return KD_EINVAL;
    const void* ptrs[] = {w->embed, w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->ffn_norm,
                          w->wg, w->wu, w->wd, w->final_norm, w->lm_head};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return fail(c, KD_EINVAL, "weight pointer NULL or not 16-byte aligned");
    const Dims& d = c->dm;
    const Layout& y = c->lay;
    cudaStream_t s = c->stream;
    const size_t D = d.d;
    KD_CUDA(c, cudaMemcpyAsync(c->arena + y.embed, w->embed, (size_t)d.V * D * 2, cudaMemcpyDeviceToDevice, s));
    KD_CUDA(c, cudaMemcpyAsync(c->arena + y.lm_head, w->lm_head, (size_t)d.V * D * 2, cudaMemcpyDeviceToDevice, s));
    KD_CUDA(c, cudaMemcpyAsync(c->arena + y.final_norm, w->final_norm, D * 2, cudaMemcpyDeviceToDevice, s));
    uint8_t* l0 = c->arena + y.layer0;
    auto per_layer = [&](size_t off, const void* src, size_t bytes) {
        return cudaMemcpy2DAsync(l0 + off, y.layer_stride, src, bytes, bytes, d.L, cudaMemcpyDeviceToDevice, s);
    };
    KD_CUDA(c, per_layer(y.l_attn_norm, w->attn_norm, D * 2));
    KD_CUDA(c, per_layer(y.l_ffn_norm, w->ffn_norm, D * 2));
    repack_qkv<<<dim3(d.qkv_rows, d.L), 128, 0, s>>>(l0, y.layer_stride, y.l_wqkv, (const uint16_t*)w->wq,
                                                      (const uint16_t*)w->wk, (const uint16_t*)w->wv, d);
    KD_CUDA(c, cudaGetLastError());
    repack_gu<<<dim3(2 * d.F, d.L), 128, 0, s>>>(l0, y.layer_stride, y.l_wgu, (const uint16_t*)w->wg,
                                                  (const uint16_t*)w->wu, d);
    KD_CUDA(c, cudaGetLastError());
    transpose_bf16<<<dim3((d.qd + 31) / 32, (d.d + 31) / 32, d.L), dim3(32, 8), 0, s>>>(
        l0, y.layer_stride, y.l_wot, (const uint16_t*)w->wo, d.d, d.qd);
    KD_CUDA(c, cudaGetLastError());
    transpose_bf16<<<dim3((d.F + 31) / 32, (d.d + 31) / 32, d.L), dim3(32, 8), 0, s>>>(
        l0, y.layer_stride, y.l_wdt, (const uint16_t*)w->wd, d.d, d.F);
    KD_CUDA(c, cudaGetLastError());
    c->launches += 4;
    // RoPE table: (cos, sin) of position p times frequency theta^(-2i/hd), formed in double
    // and rounded to float, for every position the cache can hold; the kernel reads one row
    // per step.
    {
        const int half = d.hd / 2;
        std::vector<float> tab((size_t)d.S * half * 2);
        for (int i = 0; i < half; ++i) {
            const double freq = pow((double)d.theta, -2.0 * (double)i / (double)d.hd);
            for (int pos = 0; pos < d.S; ++pos) {
                const double a = (double)pos * freq;
                tab[((size_t)pos * half + i) * 2] = (float)cos(a);
                tab[((size_t)pos * half + i) * 2 + 1] = (float)sin(a);
            }
        }
        KD_CUDA(c, cudaMemcpyAsync(c->arena + y.rope, tab.data(), tab.size() * sizeof(float), cudaMemcpyHostToDevice, s));
        KD_CUDA(c, cudaStreamSynchronize(s));  // the host table is freed on return
    }
    c->has_weights = true;
    return KD_OK;
}

int kd_set_kv(kd_ctx* c, int32_t layer, int32_t which, const void* d_src, int32_t n_pos) {
    if (!c || !d_src) return KD_EINVAL;
    const Dims& d = c->dm;
    if (layer < 0 || layer >= d.L || (which != 0 && which != 1) || n_pos < 0 || n_pos > d.S)
        return fail(c, KD_EINVAL, "kd_set_kv: bad layer/which/n_pos");
    if (n_pos == 0) return KD_OK;
    uint8_t* dst = c->arena + (which ? c->lay.vcache : c->lay.kcache) + (size_t)layer * d.Hkv * d.S * d.hd * 2;
    const size_t w = (size_t)n_pos * d.hd * 2;
    KD_CUDA(c, cudaMemcpy2DAsync(dst, (size_t)d.S * d.hd * 2, d_src, w, w, d.Hkv, cudaMemcpyDeviceToDevice,
                                 c->stream));
    return KD_OK;
}

void* kd_kv_ptr(kd_ctx* c, int32_t layer, int32_t which) {
    if (!c || layer < 0 || layer >= c->dm.L || (which != 0 && which != 1)) return nullptr;
    return c->arena + (which ? c->lay.vcache : c->lay.kcache) + (size_t)layer * c->dm.Hkv * c->dm.S * c->dm.hd * 2;
}

static int reset_common(kd_ctx* c, int32_t n_tokens, int32_t kv_len) {
    if (n_tokens < 1 || kv_len < 0 || kv_len >= c->dm.S || n_tokens > c->dm.S)
        return fail(c, KD_EINVAL, "kd_reset: need n_tokens >= 1 and 0 <= kv_len < max_seq");
    // Every completed launch leaves the control words and the split-K buffers consistent
    // (the kernel re-bases its sync count, clears its argmax slots and zeroes the buffers), so
    // they are cleared only after a failed run: the decode path then involves no memset.
    if (c->failed)
        KD_CUDA(c, cudaMemsetAsync(c->arena + c->lay.delta, 0, scratch_end(c->lay) - c->lay.delta,
                                   c->stream));
    c->pos = kv_len;
    c->n_pending = n_tokens;
    c->failed = false;
    return KD_OK;
}

int kd_reset(kd_ctx* c, const int32_t* d_tokens, int32_t n_tokens, int32_t kv_len) {
    if (!c || !d_tokens) return KD_EINVAL;
    int rc = reset_common(c, n_tokens, kv_len);
    if (rc) return rc;
    KD_CUDA(c, cudaMemcpyAsync(c->arena + c->lay.tokens_in, d_tokens, (size_t)n_tokens * 4,
                               cudaMemcpyDeviceToDevice, c->stream));
    return KD_OK;
}


int kd_decode(kd_ctx* c, int32_t n_gen, int32_t* d_tokens_out, float* d_logits_out) {
    if (!c) return KD_EINVAL;
    if (!c->has_weights || c->n_pending < 1) return fail(c, KD_ESTATE, "kd_decode: no weights or nothing pending");
    if (c->failed) return fail(c, KD_ESTATE, "kd_decode: an earlier run failed; call kd_reset");
    if (n_gen < 0 || (n_gen > 0 && !d_tokens_out)) return fail(c, KD_EINVAL, "kd_decode: bad n_gen / tokens_out");
    const int steps = c->n_pending + n_gen - 1;
    if (steps == 0) return KD_OK;
    if ((long long)c->pos + steps > c->dm.S)
        return fail(c, KD_ECAPACITY, "kd_decode: position %d + %d steps exceeds max_seq %d", c->pos, steps, c->dm.S);
    kd_ctx_view v;
    kd_internal_view(c, &v);
    Params p{};
    fill_launch_shape(v, p);
    p.arena = c->arena;
    p.lay = c->lay;
    p.steps = steps;
    p.n_pending = c->n_pending;
    p.pos0 = c->pos;
    p.n_gen = n_gen;
    p.dump = d_logits_out != nullptr;
    p.tokens_out = d_tokens_out;
    p.logits_out = d_logits_out;
    p.tag0 = c->tag;
    p.trace = c->trace;
    p.trace_every = c->trace_every;
    p.trace_rows = c->trace_rows;
    int e = 0;
    launch_decode(p, c->stream, c->smem, &e);
    if (e != 0) return fail(c, KD_ECUDA, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
    c->launches += 1;
    c->tag += (uint32_t)launch_tags(c->dm.L, steps);
    c->pos += steps;
    c->n_pending = 1;
    return KD_OK;
}

int kd_sync(kd_ctx* c) {
    if (!c) return KD_EINVAL;
    KD_CUDA(c, cudaStreamSynchronize(c->stream));
    unsigned long long st[2] = {0, 0};
    KD_CUDA(c, cudaMemcpyAsync(st, c->arena + c->lay.ctl + (size_t)kCtlStatus * 8, sizeof st,
                               cudaMemcpyDeviceToHost, c->stream));
    KD_CUDA(c, cudaStreamSynchronize(c->stream));
    if (st[0] != 0) {
        c->failed = true;
        const unsigned w = (unsigned)st[1];
        if (st[0] == (unsigned long long)kStatusToken)
            return fail(c, KD_ETOKEN, "a token id outside [0, vocab) reached the kernel at step %u", w & 0xff);
        return fail(c, KD_ETIMEOUT, "device wait exceeded its limit (kind %u, cta %u, detail %u)", w >> 24,
                    (w >> 8) & 0xffff, w & 0xff);
    }
    return KD_OK;
}

int kd_generate(kd_ctx* c, const int32_t* h_tokens, int32_t n_tokens, int32_t kv_len, int32_t n_gen,
                int32_t* h_tokens_out) {
    if (!c || !h_tokens || (n_gen > 0 && !h_tokens_out)) return KD_EINVAL;
    int rc = reset_common(c, n_tokens, kv_len);
    if (rc) return rc;
    int32_t* d_tok_out = (int32_t*)(c->arena + c->lay.tokens_out);
    KD_CUDA(c, cudaMemcpyAsync(c->arena + c->lay.tokens_in, h_tokens, (size_t)n_tokens * 4,
                               cudaMemcpyHostToDevice, c->stream));
    rc = kd_decode(c, n_gen, d_tok_out, nullptr);
    if (rc) return rc;
    if (n_gen > 0)
        KD_CUDA(c, cudaMemcpyAsync(h_tokens_out, d_tok_out, (size_t)n_gen * 4, cudaMemcpyDeviceToHost, c->stream));
    return kd_sync(c);
}

int kd_set_trace(kd_ctx* c, unsigned long long* d_buf, int64_t n_words, int32_t every) {
    if (!c) return KD_EINVAL;
    if (!d_buf) {
        c->trace = nullptr;
        return KD_OK;
    }
    if (every < 1) return fail(c, KD_EINVAL, "kd_set_trace: every must be >= 1");
    const int64_t traced = (c->nb + every - 1) / every;
    const int64_t rows = n_words / (traced * kTraceWords);
    if (rows < 2 || rows > (1 << 30)) return fail(c, KD_EINVAL, "kd_set_trace: buffer too small");
    c->trace = d_buf;
    c->trace_every = every;
    c->trace_rows = (int)rows;
    return KD_OK;
}

int kd_set_sampling(kd_ctx* c, float temperature, uint64_t seed) {
    if (!c) return KD_EINVAL;
    if (!(temperature >= 0.0f) || !isfinite(temperature))
        return fail(c, KD_EINVAL, "kd_set_sampling: temperature must be finite and >= 0");
    c->inv_temp = temperature > 0.0f ? 1.0f / temperature : 0.0f;
    c->seed = seed;
    return KD_OK;
}

int kd_set_timeout(kd_ctx* c, int64_t ns) {
    if (!c || ns < 1) return KD_EINVAL;
    c->timeout_ns = ns;
    return KD_OK;
}

int32_t kd_position(const kd_ctx* c) { return c ? c->pos : -1; }

int kd_get_info(const kd_ctx* c, kd_info* info) {
    if (!c || !info) return KD_EINVAL;
    info->grid = c->nb;
    info->threads = kThreads;
    info->smem_bytes = c->smem;
    info->stages = c->ns;
    info->stage_bytes = kStageBytes;
    info->attn_pieces = c->pieces;
    info->arena_bytes = (int64_t)c->lay.total;
    info->weight_bytes = (int64_t)c->lay.weights_end;
    info->kv_bytes = (int64_t)c->lay.kv_bytes;
    info->launches = c->launches;
    info->ctl_offset = (int64_t)c->lay.ctl;
    info->sync_replicas = c->nsync;
    info->sync_offset[0] = (int64_t)c->sync_off[0];
    info->sync_offset[1] = (int64_t)c->sync_off[1];
    return KD_OK;
}

const char* kd_last_error(const kd_ctx* c) { return c ? c->err : "no handle"; }

const char* kd_strerror(int code) {
    switch (code) {
        case KD_OK: return "ok";
        case KD_EINVAL: return "invalid argument or unsupported configuration";
        case KD_ENOMEM: return "arena too small or misaligned";
        case KD_ECAPACITY: return "KV capacity (max_seq) exceeded";
        case KD_ECOOP: return "kernel cannot be co-resident on every SM";
        case KD_ECUDA: return "CUDA runtime error";
        case KD_ETIMEOUT: return "device-side wait exceeded its limit";
        case KD_ESTATE: return "call out of order";
        case KD_ETOKEN: return "token id outside the vocabulary";
        default: return "unknown error";
    }
}

void kd_destroy(kd_ctx* c) { free(c); }

}  // extern "C"
