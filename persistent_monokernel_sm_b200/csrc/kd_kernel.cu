// kd_kernel.cu -- the decode monokernel: one persistent cooperative launch per kd_decode
// that runs every decode step of the request, layer after layer, without returning to the
// host ("3000 tokens per second: how to speed up LLMs on ordinary GPUs", aikraft.ru,
// section 04 "Monokernel and optimized GPU code": one resident GPU program covering matrix
// products, attention, normalisation and sampling, with tight control of synchronisation,
// prefetch and execution order).
//
// B200 design (one CTA per SM, 148 CTAs):
//  * Warp specialisation. Warp 8 of each CTA is the producer: one lane walks the CTA's
//    fixed schedule of weight tiles (and KV-cache tiles) and streams them HBM -> shared
//    memory with 1-D bulk async copies (cp.async.bulk) into a ring of 32 KB stages guarded
//    by mbarriers. Warps 0-7 are consumers; ring slot i belongs to consumer warp i, which
//    takes each stage that lands there whole. (A parity wait on an mbarrier can only tell
//    the current phase from the one before it, so the warp that waits on a slot must be
//    the one that finished the slot's previous stage.)
//  * Weights never depend on activations, so the producer keeps streaming while the
//    consumers wait at a grid barrier: the ring absorbs barrier latency instead of leaving
//    HBM idle (the pages name prefetch and synchronisation control as the monokernel's
//    levers, aikraft.ru section 04; the per-token time budget that makes each microsecond
//    count is their section 03).
//  * Batch-1 decode is a matrix-vector product (about 1 FLOP per weight byte, their
//    section 02), so there are no tensor-core tiles: 16-byte bf16 loads from shared
//    memory, fp32 FMAs, warp-shuffle reductions.
//  * Phases of a layer are separated by grid barriers built on a monotonic device-scope
//    arrival counter (release add / acquire poll); every wait is time-limited and unwinds
//    with an error status instead of hanging.
//  * Attention is split-K over the KV positions (CTAs per kv head x position pieces) with
//    an online-softmax state per warp, merged per CTA, and combined across CTAs by the
//    last-arriving CTA of each kv head.
//  * The LM head ends in a packed (value, index) atomicMax; every CTA reads the winner
//    and gathers the next embedding row itself, so sampling never leaves the GPU
//    (agentlenshq.com "Breaking the memory wall", section "1. The Monokernel Runtime").
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "kd_layout.h"

namespace kd {

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(a),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, "
        "[%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(mbar), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ uint64_t ld_acquire_u64(const unsigned long long* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, uint64_t v) {
    asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
}
// Consumer-wide barrier that also ANDs a per-thread flag across the consumer warps.
__device__ __forceinline__ bool consumer_sync_and(bool v) {
    uint32_t r;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, 1, %2, p; selp.u32 %0, 1, 0, q; }"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kConsumerThreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ int read_status(const unsigned long long* ctl) {
    return static_cast<int>(*reinterpret_cast<const volatile unsigned long long*>(ctl + kCtlStatus));
}
__device__ __noinline__ void raise_timeout(unsigned long long* ctl, int where) {
    if (atomicCAS(ctl + kCtlStatus, 0ull, (unsigned long long)kStatusTimeout) == 0ull)
        atomicExch(ctl + kCtlWhere, (unsigned long long)where);
}

// Where a wait gave up: (what << 24) | (cta << 8) | detail.
enum { kWhereFull = 1, kWhereEmpty = 2, kWhereGrid = 3, kWhereKv = 4 };
__device__ __forceinline__ int where_code(int what, int detail) {
    return (what << 24) | ((int)blockIdx.x << 8) | (detail & 0xff);
}

// Optional per-phase timestamps (SM cycles) of one CTA, recorded by consumer thread 0.
struct Tracer {
    unsigned long long* row0 = nullptr;
    int row = 0, rows = 0;
    __device__ void mark(int col) {
        if (row0 && row < rows - 1) row0[(size_t)row * kTraceWords + col] = (unsigned long long)clock64();
    }
    __device__ void next() { ++row; }
};

// ------------------------------------------------------------------ schedule geometry
// Both the producer and the consumers enumerate the same stage sequence from these.

enum Phase { kQKV = 0, kATT = 1, kO = 2, kGU = 3, kD = 4, kLM = 5 };

struct Gemv {
    const uint8_t* base;  // matrix rows
    int K;                // reduction length (bf16 elements per row)
    int row0, row1;       // this CTA's rows
    int R;                // rows per stage
};

__device__ __forceinline__ Gemv gemv_geom(const Params& P, int phase, int l, int c) {
    const Dims& dm = P.dm;
    const uint8_t* lb = P.arena + P.lay.layer0 + (size_t)l * P.lay.layer_stride;
    Gemv g;
    int units, rpu;
    switch (phase) {
        case kQKV: g.base = lb + P.lay.l_wqkv; g.K = dm.d; units = dm.qkv_rows / 2; rpu = 2; g.R = P.rows_qkv; break;
        case kO: g.base = lb + P.lay.l_wo; g.K = dm.qd; units = dm.d; rpu = 1; g.R = P.rows_o; break;
        case kGU: g.base = lb + P.lay.l_wgu; g.K = dm.d; units = dm.F; rpu = 2; g.R = P.rows_gu; break;
        case kD: g.base = lb + P.lay.l_wd; g.K = dm.F; units = dm.d; rpu = 1; g.R = P.rows_d; break;
        default: g.base = P.arena + P.lay.lm_head; g.K = dm.d; units = dm.V; rpu = 1; g.R = P.rows_lm; break;
    }
    g.row0 = (int)((long long)units * c / P.nb) * rpu;
    g.row1 = (int)((long long)units * (c + 1) / P.nb) * rpu;
    return g;
}
__device__ __forceinline__ int gemv_stages(const Gemv& g) { return (g.row1 - g.row0 + g.R - 1) / g.R; }

struct Attn {
    int g, piece;  // kv head, piece index (g < 0: this CTA has no piece)
    int a, b;      // positions [a, b) of the piece (b may include the current position)
    int tma_end;   // [a, tma_end) streamed through the ring; position p handled directly
};

__device__ __forceinline__ Attn attn_geom(const Params& P, int p, int c) {
    Attn at;
    const int A = P.attn_pieces;
    if (c >= A * P.dm.Hkv) {
        at.g = -1;
        at.piece = 0;
        at.a = at.b = at.tma_end = 0;
        return at;
    }
    at.g = c / A;
    at.piece = c % A;
    const long long T = (long long)p + 1;
    at.a = (int)(T * at.piece / A);
    at.b = (int)(T * (at.piece + 1) / A);
    at.tma_end = at.b < p ? at.b : p;
    if (at.tma_end < at.a) at.tma_end = at.a;
    return at;
}
__device__ __forceinline__ int attn_stages(const Params& P, const Attn& at) {
    return (at.tma_end - at.a + P.pos_per_stage - 1) / P.pos_per_stage;
}

// The LM head runs at steps that pick a token, or at every step when logits are dumped.
__device__ __forceinline__ bool step_has_head(const Params& P, int t) {
    return P.dump || t >= P.n_pending - 1;
}
// Grid barriers completed before step s begins.
__device__ __forceinline__ long long barriers_before_step(const Params& P, int s) {
    long long heads = P.dump ? s : (s - (P.n_pending - 1) > 0 ? s - (P.n_pending - 1) : 0);
    return (long long)s * 5 * P.dm.L + heads;
}

// ------------------------------------------------------------------ shared memory

struct Smem {
    uint8_t* ring;          // ns * kStageBytes
    float* xs;              // activation vector in split layout / attention merge scratch
    float* qs;              // attention q (r * hd)
    float2* rope;           // (cos, sin) for hd/2 frequencies at this step's position
    float* red;             // reduction scratch
    unsigned long long* best;  // per-warp argmax keys
    int* flag;              // broadcast slots
    uint64_t* full;         // mbarriers
    uint64_t* empty;
    float* sp;              // per-stage partial sums [slot][phase][row * KS + slice] (16 each)
    int* scnt;              // per-stage arrival counts [slot][phase]
};

__device__ __forceinline__ Smem carve(const Params& P, uint8_t* base) {
    Smem s;
    size_t off = 0;
    s.ring = base;
    off += (size_t)P.ns * kStageBytes;
    s.xs = reinterpret_cast<float*>(base + off);
    off += (size_t)P.xs_floats * 4;
    s.qs = reinterpret_cast<float*>(base + off);
    off += (size_t)kMaxGroup * 128 * 4;
    s.rope = reinterpret_cast<float2*>(base + off);
    off += 64 * 8;
    s.red = reinterpret_cast<float*>(base + off);
    off += 64 * 4;
    s.best = reinterpret_cast<unsigned long long*>(base + off);
    off += kConsumerWarps * 8;
    s.flag = reinterpret_cast<int*>(base + off);
    off += 16 * 4;
    s.full = reinterpret_cast<uint64_t*>(base + off);
    off += kMaxStages * 8;
    s.empty = reinterpret_cast<uint64_t*>(base + off);
    off += kMaxStages * 8;
    s.sp = reinterpret_cast<float*>(base + off);
    off += (size_t)kMaxStages * 2 * kMaxRows * 4;
    s.scnt = reinterpret_cast<int*>(base + off);
    return s;
}

int monokernel_smem_bytes(const Params& p) {
    return p.ns * kStageBytes + p.xs_floats * 4 + kMaxGroup * 128 * 4 + 64 * 8 + 64 * 4 +
           kConsumerWarps * 8 + 16 * 4 + 2 * kMaxStages * 8 + kMaxStages * 2 * kMaxRows * 4 +
           kMaxStages * 2 * 4;
}

// Split layout of an activation vector of length K (K % 8 == 0): element k lives at
// ((k & 7) >> 2) * (K / 2) + (k >> 3) * 4 + (k & 3), so lane-strided 8-element chunks
// read as two conflict-free float4 loads.
__device__ __forceinline__ int xs_index(int k, int K) {
    return ((k & 7) >> 2) * (K >> 1) + ((k >> 3) << 2) + (k & 3);
}

// ------------------------------------------------------------------ waits

// Position in the stage sequence: stage k lives in ring slot k % ns; `phase` is the parity
// of the slot's current use (it flips each time the ring wraps).
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void advance(int ns) {
        if (++slot == ns) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// Parity wait with a hardware suspend hint: the warp sleeps until the phase completes
// instead of spinning; every few wake-ups it checks the abort flag and its time limit.
__device__ __forceinline__ bool mbar_wait_hint(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(a), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}

__device__ bool wait_full(const Smem& sm, const Ring& rg, const Params& P, unsigned long long* ctl) {
    const uint32_t a = smem_u32(&sm.full[rg.slot]);
    if (__all_sync(0xffffffffu, mbar_try_wait(a, rg.phase))) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (__all_sync(0xffffffffu, mbar_wait_hint(a, rg.phase))) return true;
        int bad = 0;
        if ((threadIdx.x & 31) == 0) {
            bad = read_status(ctl) != 0;
            if (!bad && globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                raise_timeout(ctl, where_code(kWhereFull, rg.slot));
                bad = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, bad, 0)) return false;
    }
}

// Grid-wide barrier among the consumer warps of all CTAs. `epoch` counts barriers this
// launch has completed; arrivals accumulate in one monotonic counter, so there is no
// reset race and a barrier completes when the counter reaches base + epoch * nb.
// `local_ok` is false in a warp whose wait gave up; the result is the same for every
// consumer thread of the CTA, and false in every CTA once any wait anywhere has given up
// (the device status word is re-read after the barrier completes).
__device__ bool grid_sync(const Smem& sm, long long& epoch, uint64_t base, const Params& P,
                          unsigned long long* ctl, bool local_ok, Tracer& tr) {
    // every consumer warp's writes of this phase are done; did every warp succeed?
    const bool cta_ok = consumer_sync_and(local_ok);
    if (threadIdx.x == 0) tr.mark(2);
    if (threadIdx.x == 0 && !cta_ok) sm.flag[0] = 0;
    if (threadIdx.x == 0 && cta_ok) {
        __threadfence();
        red_release_add_u64(ctl + kCtlBar, 1ull);
        const uint64_t target = base + (uint64_t)(epoch + 1) * (uint64_t)P.nb;
        int ok = 1;
        if (ld_acquire_u64(ctl + kCtlBar) < target) {
            const uint64_t t0 = globaltimer();
            for (uint32_t it = 0;; ++it) {
                if (ld_acquire_u64(ctl + kCtlBar) >= target) break;
                if ((it & 31) == 31) {
                    if (read_status(ctl) != 0) { ok = 0; break; }
                    if (globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                        raise_timeout(ctl, where_code(kWhereGrid, (int)(epoch & 0xff)));
                        ok = 0;
                        break;
                    }
                }
            }
        }
        __threadfence();
        if (ok && read_status(ctl) != 0) ok = 0;
        sm.flag[0] = ok;
        tr.mark(3);
        tr.next();
        tr.mark(0);
    }
    consumer_sync();
    ++epoch;
    return sm.flag[0] != 0;
}

// ------------------------------------------------------------------ activation loads

// xs <- x * rsqrt(mean(x^2) + eps) * g in split layout. src_f32 (global, written during
// the launch) or src_bf16 (an embedding row, read-only).
__device__ void load_rmsnorm(const Smem& sm, const float* src_f32, const __nv_bfloat16* src_bf16,
                             const __nv_bfloat16* gain, int K, float eps) {
    const int tid = threadIdx.x;
    float ss = 0.f;
    for (int k = tid * 4; k < K; k += kConsumerThreads * 4) {
        float4 v;
        if (src_f32) {
            v = __ldcg(reinterpret_cast<const float4*>(src_f32 + k));
        } else {
            const uint2 w = __ldg(reinterpret_cast<const uint2*>(src_bf16 + k));
            v = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
        }
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        *reinterpret_cast<float4*>(&sm.xs[xs_index(k, K)]) = v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) sm.red[tid >> 5] = ss;
    consumer_sync();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += sm.red[w];
    const float inv = 1.0f / sqrtf(tot / (float)K + eps);
    for (int k = tid * 4; k < K; k += kConsumerThreads * 4) {
        float4* p = reinterpret_cast<float4*>(&sm.xs[xs_index(k, K)]);
        const uint2 gw = __ldg(reinterpret_cast<const uint2*>(gain + k));
        float4 v = *p;
        v.x = (v.x * inv) * bf_lo(gw.x);
        v.y = (v.y * inv) * bf_hi(gw.x);
        v.z = (v.z * inv) * bf_lo(gw.y);
        v.w = (v.w * inv) * bf_hi(gw.y);
        *p = v;
    }
    consumer_sync();
}

__device__ void load_vector(const Smem& sm, const float* src, int K) {
    for (int k = threadIdx.x * 4; k < K; k += kConsumerThreads * 4)
        *reinterpret_cast<float4*>(&sm.xs[xs_index(k, K)]) = __ldcg(reinterpret_cast<const float4*>(src + k));
    consumer_sync();
}

// ------------------------------------------------------------------ GEMV stage

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xffffffffu - (uint32_t)idx);
}
__device__ __forceinline__ int key_index(unsigned long long key) {
    return (int)(0xffffffffu - (uint32_t)(key & 0xffffffffull));
}

struct StepCtx {
    int t, p, l;
    unsigned long long lm_best;  // running argmax key of this warp (lane 0)
};

// Partial dot products of one warp's share of a stage: rows [ra, ra + nr) (nr <= 2) over
// the 8-element chunks [c0, c1) of the row, lane-strided; returns the warp-reduced sums.
__device__ __forceinline__ void gemv_part(const uint8_t* st, size_t rowb, int ra, int nr, int c0, int c1,
                                          const float* xs, int K, float& s0, float& s1) {
    const int lane = threadIdx.x & 31;
    float a0 = 0.f, b0 = 0.f, a1 = 0.f, b1 = 0.f;
    const float4* xlo = reinterpret_cast<const float4*>(xs);
    const float4* xhi = reinterpret_cast<const float4*>(xs + (K >> 1));
    const uint8_t* w0 = st + (size_t)ra * rowb;
    const uint8_t* w1 = w0 + rowb;
    if (nr == 2) {
#pragma unroll 4
        for (int c = c0 + lane; c < c1; c += 32) {
            const float4 x = xlo[c], y = xhi[c];
            const uint4 p = *reinterpret_cast<const uint4*>(w0 + (size_t)c * 16);
            const uint4 q = *reinterpret_cast<const uint4*>(w1 + (size_t)c * 16);
            a0 = fmaf(bf_lo(p.x), x.x, a0); b0 = fmaf(bf_hi(p.x), x.y, b0);
            a0 = fmaf(bf_lo(p.y), x.z, a0); b0 = fmaf(bf_hi(p.y), x.w, b0);
            a0 = fmaf(bf_lo(p.z), y.x, a0); b0 = fmaf(bf_hi(p.z), y.y, b0);
            a0 = fmaf(bf_lo(p.w), y.z, a0); b0 = fmaf(bf_hi(p.w), y.w, b0);
            a1 = fmaf(bf_lo(q.x), x.x, a1); b1 = fmaf(bf_hi(q.x), x.y, b1);
            a1 = fmaf(bf_lo(q.y), x.z, a1); b1 = fmaf(bf_hi(q.y), x.w, b1);
            a1 = fmaf(bf_lo(q.z), y.x, a1); b1 = fmaf(bf_hi(q.z), y.y, b1);
            a1 = fmaf(bf_lo(q.w), y.z, a1); b1 = fmaf(bf_hi(q.w), y.w, b1);
        }
    } else if (nr == 1) {
#pragma unroll 4
        for (int c = c0 + lane; c < c1; c += 32) {
            const float4 x = xlo[c], y = xhi[c];
            const uint4 p = *reinterpret_cast<const uint4*>(w0 + (size_t)c * 16);
            a0 = fmaf(bf_lo(p.x), x.x, a0); b0 = fmaf(bf_hi(p.x), x.y, b0);
            a0 = fmaf(bf_lo(p.y), x.z, a0); b0 = fmaf(bf_hi(p.y), x.w, b0);
            a0 = fmaf(bf_lo(p.z), y.x, a0); b0 = fmaf(bf_hi(p.z), y.y, b0);
            a0 = fmaf(bf_lo(p.w), y.z, a0); b0 = fmaf(bf_hi(p.w), y.w, b0);
        }
    }
    s0 = a0 + b0;
    s1 = a1 + b1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
}

// One GEMV phase. Every consumer warp takes part in every stage: the stage's R rows are
// split into RG row groups x KS column slices (RG * KS = 8 warps, at most 2 rows per
// warp), each warp writes its partial sums to shared memory, and the last warp to finish
// the stage adds the KS slices in a fixed order and applies the phase's epilogue.
// A wait that gives up marks `ok` false and the warp skips the work of the remaining
// stages, but it still reaches every named barrier; the next grid barrier then reports
// the failure to the whole CTA at once.
__device__ void run_gemv(const Params& P, const Smem& sm, unsigned long long* ctl, int phase, int l,
                         Ring& rg, StepCtx& sc, bool& ok) {
    const Dims& dm = P.dm;
    const Gemv g = gemv_geom(P, phase, l, blockIdx.x);
    const int nst = gemv_stages(g);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int RG = g.R >= 8 ? 8 : (g.R >= 4 ? 4 : (g.R >= 2 ? 2 : 1));
    const int KS = kConsumerWarps / RG;
    const int grp = warp / KS, ks = warp % KS;
    const int nch = g.K >> 3;
    const int c0 = nch * ks / KS, c1 = nch * (ks + 1) / KS;
    const size_t rowb = (size_t)g.K * 2;
    float* xg = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.x);
    for (int j = 0; j < nst; ++j, rg.advance(P.ns)) {
        if (!ok) continue;
        if (!wait_full(sm, rg, P, ctl)) {
            ok = false;
            continue;
        }
        const int r0 = g.row0 + j * g.R;
        const int n = min(g.R, g.row1 - r0);
        const int ra = n * grp / RG, nr = n * (grp + 1) / RG - ra;
        float s0, s1;
        gemv_part(sm.ring + (size_t)rg.slot * kStageBytes, rowb, ra, nr, c0, c1, sm.xs, g.K, s0, s1);
        __syncwarp();
        // rows * KS <= kMaxRows for every split (R >= 8 -> KS = 1; R < 8 -> R * KS < 16)
        float* sp = sm.sp + (size_t)(rg.slot * 2 + rg.phase) * kMaxRows;
        int* cnt = sm.scnt + rg.slot * 2 + rg.phase;
        int last = 0;
        if (lane == 0) {
            mbar_arrive(smem_u32(&sm.empty[rg.slot]));  // this warp is done reading the stage
            if (nr > 0) sp[ra * KS + ks] = s0;
            if (nr > 1) sp[(ra + 1) * KS + ks] = s1;
            __threadfence_block();
            last = atomicAdd(cnt, 1) == kConsumerWarps - 1;
        }
        if (!__shfl_sync(0xffffffffu, last, 0)) continue;
        // ---- last warp of this stage: row totals (lane = row) and the epilogue
        __threadfence_block();
        float tot = 0.f;
        if (lane < n)
            for (int q = 0; q < KS; ++q) tot += sp[lane * KS + q];
        if (lane == 0) *cnt = 0;
        if (phase == kQKV || phase == kGU) {
            const float nb = __shfl_down_sync(0xffffffffu, tot, 1);
            if (!(lane & 1) && lane < n) {
                const float a = tot, b = nb;
                const int row = r0 + lane;  // even row of a (RoPE pair | gate, up) pair
                if (phase == kGU) {
                    float* hdn = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.hdn);
                    __stcg(hdn + (row >> 1), a / (1.0f + expf(-a)) * b);
                } else if (row < dm.qd + dm.kvd) {
                    const int hd = dm.hd;
                    const bool isq = row < dm.qd;
                    const int rr = isq ? row : row - dm.qd;
                    const int h = rr / hd, i = (rr % hd) >> 1;
                    const float2 cs = sm.rope[i];
                    const float ra_ = a * cs.x - b * cs.y;
                    const float rb_ = b * cs.x + a * cs.y;
                    if (isq) {
                        float* q = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.q);
                        __stcg(q + h * hd + i, ra_);
                        __stcg(q + h * hd + i + hd / 2, rb_);
                    } else {
                        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.kcache) +
                                            (((size_t)l * dm.Hkv + h) * dm.S + sc.p) * hd;
                        kc[i] = __float2bfloat16_rn(ra_);
                        kc[i + hd / 2] = __float2bfloat16_rn(rb_);
                        fence_proxy_async_global();
                    }
                } else {
                    const int rr = row - dm.qd - dm.kvd;
                    const int h = rr / dm.hd, j2 = rr % dm.hd;
                    __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.vcache) +
                                        (((size_t)l * dm.Hkv + h) * dm.S + sc.p) * dm.hd;
                    vc[j2] = __float2bfloat16_rn(a);
                    vc[j2 + 1] = __float2bfloat16_rn(b);
                    fence_proxy_async_global();
                }
            }
        } else if (phase == kO || phase == kD) {
            if (lane < n) __stcg(xg + r0 + lane, __ldcg(xg + r0 + lane) + tot);
        } else {  // LM head: dump, then this warp's running argmax (lowest index on ties)
            if (P.dump && lane < n) __stcg(P.logits_out + (size_t)sc.t * dm.V + r0 + lane, tot);
            unsigned long long key = lane < n ? argmax_key(tot, r0 + lane) : 0ull;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
                key = other > key ? other : key;
            }
            if (lane == 0 && key > sc.lm_best) sc.lm_best = key;
        }
    }
}

// ------------------------------------------------------------------ attention phase

template <int HD>
__device__ void run_attention(const Params& P, const Smem& sm, unsigned long long* ctl, int l, Ring& rg,
                              StepCtx& sc, bool& ok) {
    constexpr int E = HD / 32;  // dims per lane
    const Dims& dm = P.dm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const Attn at = attn_geom(P, sc.p, blockIdx.x);
    if (at.g < 0) return;  // uniform across the CTA
    const int r = dm.r, A = P.attn_pieces;
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
    const float* qg = reinterpret_cast<const float*>(P.arena + P.lay.q) + (size_t)at.g * r * HD;
    for (int i = tid; i < r * HD; i += kConsumerThreads) sm.qs[i] = __ldcg(qg + i) * qscale;
    consumer_sync();

    float q[kMaxGroup][E], m[kMaxGroup], lsum[kMaxGroup], acc[kMaxGroup][E];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        m[h] = -INFINITY;
        lsum[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            acc[h][e] = 0.f;
            q[h][e] = h < r ? sm.qs[h * HD + lane * E + e] : 0.f;
        }
    }
    auto visit = [&](const __nv_bfloat16* krow, const __nv_bfloat16* vrow, bool global) {
        float kv[E], vv[E];
        if constexpr (E == 4) {
            uint2 kw, vw;
            if (global) {
                kw = __ldcg(reinterpret_cast<const uint2*>(krow + lane * E));
                vw = __ldcg(reinterpret_cast<const uint2*>(vrow + lane * E));
            } else {
                kw = *reinterpret_cast<const uint2*>(krow + lane * E);
                vw = *reinterpret_cast<const uint2*>(vrow + lane * E);
            }
            kv[0] = bf_lo(kw.x), kv[1] = bf_hi(kw.x), kv[2] = bf_lo(kw.y), kv[3] = bf_hi(kw.y);
            vv[0] = bf_lo(vw.x), vv[1] = bf_hi(vw.x), vv[2] = bf_lo(vw.y), vv[3] = bf_hi(vw.y);
        } else {
            uint32_t kw, vw;
            if (global) {
                kw = __ldcg(reinterpret_cast<const unsigned int*>(krow + lane * E));
                vw = __ldcg(reinterpret_cast<const unsigned int*>(vrow + lane * E));
            } else {
                kw = *reinterpret_cast<const uint32_t*>(krow + lane * E);
                vw = *reinterpret_cast<const uint32_t*>(vrow + lane * E);
            }
            kv[0] = bf_lo(kw), kv[1] = bf_hi(kw);
            vv[0] = bf_lo(vw), vv[1] = bf_hi(vw);
        }
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < r) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) s = fmaf(q[h][e], kv[e], s);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                const float mn = fmaxf(m[h], s);
                const float corr = exp2f(m[h] - mn);
                const float pr = exp2f(s - mn);
                lsum[h] = lsum[h] * corr + pr;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] = fmaf(acc[h][e], corr, pr * vv[e]);
                m[h] = mn;
            }
        }
    };

    // every warp takes an eighth of each stage's positions and keeps its own softmax state
    const int nst = attn_stages(P, at);
    for (int j = 0; j < nst; ++j, rg.advance(P.ns)) {
        if (!ok) continue;
        if (!wait_full(sm, rg, P, ctl)) {
            ok = false;
            continue;
        }
        const int s0 = at.a + j * P.pos_per_stage;
        const int n = min(P.pos_per_stage, at.tma_end - s0);
        const __nv_bfloat16* st = reinterpret_cast<const __nv_bfloat16*>(sm.ring + (size_t)rg.slot * kStageBytes);
        const __nv_bfloat16* vst = st + (size_t)n * HD;
        const int p0 = n * warp / kConsumerWarps, p1 = n * (warp + 1) / kConsumerWarps;
        for (int jj = p0; jj < p1; ++jj) visit(st + (size_t)jj * HD, vst + (size_t)jj * HD, false);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.empty[rg.slot]));
    }
    // the current position, written by this step's QKV phase, read straight from the cache
    if (at.b > sc.p && warp == kConsumerWarps - 1) {
        const size_t off = (((size_t)l * dm.Hkv + at.g) * dm.S + sc.p) * HD;
        visit(reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.kcache) + off,
              reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.vcache) + off, true);
    }

    // merge the warps' states (xs is free during attention)
    const int rec = HD + 2;
    float* ws = sm.xs;  // [warp][h][rec]
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h < r) {
            float* wr = ws + ((size_t)warp * r + h) * rec;
            if (lane == 0) wr[0] = m[h], wr[1] = lsum[h];
#pragma unroll
            for (int e = 0; e < E; ++e) wr[2 + lane * E + e] = acc[h][e];
        }
    }
    consumer_sync();
    float* part = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.part);
    float* mine = part + ((size_t)(at.g * A + at.piece) * r) * rec;
    for (int idx = tid; idx < r * HD; idx += kConsumerThreads) {
        const int h = idx / HD, dd = idx % HD;
        float M = -INFINITY;
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ws[((size_t)w * r + h) * rec]);
        float L = 0.f, o = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float* wr = ws + ((size_t)w * r + h) * rec;
                if (wr[0] == -INFINITY) continue;
                const float f = exp2f(wr[0] - M);
                L = fmaf(wr[1], f, L);
                o = fmaf(wr[2 + dd], f, o);
            }
        }
        if (dd == 0) __stcg(mine + (size_t)h * rec, M), __stcg(mine + (size_t)h * rec + 1, L);
        __stcg(mine + (size_t)h * rec + 2 + dd, o);
    }
    consumer_sync();
    if (tid == 0) {
        __threadfence();
        unsigned int* cnt = reinterpret_cast<unsigned int*>(ctl + kCtlHead + 16 * at.g);
        const unsigned int old = atomicAdd(cnt, 1u);
        sm.flag[1] = ((old + 1u) % (unsigned)A) == 0u;
        __threadfence();
    }
    consumer_sync();
    if (sm.flag[1]) {  // last piece of this kv head to finish: combine all pieces
        float* og = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.o) + (size_t)at.g * r * HD;
        const float* hp = part + (size_t)at.g * A * r * rec;
        for (int idx = tid; idx < r * HD; idx += kConsumerThreads) {
            const int h = idx / HD, dd = idx % HD;
            float M = -INFINITY;
            for (int i = 0; i < A; ++i) M = fmaxf(M, __ldcg(hp + ((size_t)i * r + h) * rec));
            float L = 0.f, o = 0.f;
            for (int i = 0; i < A; ++i) {
                const float* pr = hp + ((size_t)i * r + h) * rec;
                const float mi = __ldcg(pr);
                if (mi == -INFINITY) continue;
                const float f = exp2f(mi - M);
                L = fmaf(__ldcg(pr + 1), f, L);
                o = fmaf(__ldcg(pr + 2 + dd), f, o);
            }
            __stcg(og + (size_t)h * HD + dd, o / L);
        }
    }
}

// ------------------------------------------------------------------ producer

struct Producer {
    const Params& P;
    const Smem& sm;
    unsigned long long* ctl;
    uint64_t base;
    uint64_t policy;
    int k = 0;              // stages issued
    int slot = 0, pass = 0;  // ring position of stage k: slot k % ns, pass k / ns
    long long seen_epochs = 0;
    unsigned long long wait_slot = 0, wait_kv = 0;  // cycles blocked (trace)

    __device__ Producer(const Params& p, const Smem& s, unsigned long long* c, uint64_t b)
        : P(p), sm(s), ctl(c), base(b) {
        policy = policy_evict_first();
    }

    // Wait until every consumer warp has released the previous stage in this slot.
    __device__ bool wait_empty() {
        if (pass == 0) return true;
        const uint32_t a = smem_u32(&sm.empty[slot]);
        const uint32_t par = (uint32_t)((pass - 1) & 1);
        if (mbar_try_wait(a, par)) return true;
        const uint64_t t0 = globaltimer();
        const long long c0 = clock64();
        for (;;) {
            if (mbar_wait_hint(a, par)) {
                wait_slot += (unsigned long long)(clock64() - c0);
                return true;
            }
            if (read_status(ctl) != 0) return false;
            if (globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                raise_timeout(ctl, where_code(kWhereEmpty, slot));
                return false;
            }
        }
    }

    // Wait until at least `need` grid barriers of this launch have completed.
    __device__ bool wait_epochs(long long need) {
        if (seen_epochs >= need) return true;
        const uint64_t t0 = globaltimer();
        const long long c0 = clock64();
        for (uint32_t it = 0;; ++it) {
            seen_epochs = (long long)((ld_acquire_u64(ctl + kCtlBar) - base) / (uint64_t)P.nb);
            if (seen_epochs >= need) break;
            if ((it & 31) == 31) {
                if (read_status(ctl) != 0) return false;
                if (globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                    raise_timeout(ctl, where_code(kWhereKv, 0));
                    return false;
                }
            }
        }
        wait_kv += (unsigned long long)(clock64() - c0);
        fence_proxy_async_global();
        return true;
    }

    __device__ bool issue(const void* src, uint32_t bytes, const void* src2, uint32_t bytes2) {
        if (!wait_empty()) return false;
        const uint32_t fb = smem_u32(&sm.full[slot]);
        const uint32_t dst = smem_u32(sm.ring + (size_t)slot * kStageBytes);
        mbar_expect_tx(fb, bytes + bytes2);
        bulk_g2s(dst, src, bytes, fb, policy);
        if (bytes2) bulk_g2s(dst + bytes, src2, bytes2, fb, policy);
        ++k;
        if (++slot == P.ns) {
            slot = 0;
            ++pass;
        }
        return true;
    }

    __device__ bool gemv(int phase, int l) {
        const Gemv g = gemv_geom(P, phase, l, blockIdx.x);
        const size_t rowb = (size_t)g.K * 2;
        for (int r0 = g.row0; r0 < g.row1; r0 += g.R) {
            const int n = min(g.R, g.row1 - r0);
            if (!issue(g.base + (size_t)r0 * rowb, (uint32_t)(n * rowb), nullptr, 0)) return false;
        }
        return true;
    }

    __device__ bool attention(int t, int l) {
        const int p = P.pos0 + t;
        const Attn at = attn_geom(P, p, blockIdx.x);
        if (at.g < 0) return true;
        const Dims& dm = P.dm;
        const size_t head = ((size_t)l * dm.Hkv + at.g) * dm.S;
        const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.kcache);
        const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.vcache);
        for (int s0 = at.a; s0 < at.tma_end; s0 += P.pos_per_stage) {
            const int n = min(P.pos_per_stage, at.tma_end - s0);
            const int last = s0 + n - 1;
            if (last >= P.pos0) {  // written earlier in this launch: wait for its QKV barrier
                const long long need = barriers_before_step(P, last - P.pos0) + 5ll * l + 1;
                if (!wait_epochs(need)) return false;
            }
            const uint32_t bytes = (uint32_t)((size_t)n * dm.hd * 2);
            if (!issue(kc + (head + s0) * dm.hd, bytes, vc + (head + s0) * dm.hd, bytes)) return false;
        }
        return true;
    }

    __device__ void run() {
        const long long c_start = clock64();
        bool ok = true;
        for (int t = 0; t < P.steps && ok; ++t) {
            for (int l = 0; l < P.dm.L && ok; ++l) {
                ok = gemv(kQKV, l) && attention(t, l) && gemv(kO, l) && gemv(kGU, l) && gemv(kD, l);
            }
            if (ok && step_has_head(P, t)) ok = gemv(kLM, 0);
        }
        if (!ok) {
            // unwinding: let every copy already issued land before the CTA exits
            const int first = k > P.ns ? k - P.ns : 0;
            for (int kk = first; kk < k; ++kk) {
                const uint32_t a = smem_u32(&sm.full[kk % P.ns]);
                const uint32_t par = (uint32_t)((kk / P.ns) & 1);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(a, par) && globaltimer() - t0 < (uint64_t)P.timeout_ns) {
                }
            }
        }
        if (P.trace && blockIdx.x % P.trace_every == 0) {
            unsigned long long* r = P.trace + ((size_t)(blockIdx.x / P.trace_every) * P.trace_rows + P.trace_rows - 1) * kTraceWords;
            r[0] = wait_slot, r[1] = wait_kv, r[2] = (unsigned long long)k;
            r[3] = (unsigned long long)(clock64() - c_start);
        }
    }
};

// ------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, 1) monokernel(const __grid_constant__ Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem sm = carve(P, smem_raw);
    unsigned long long* ctl = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.ctl);
    const int tid = threadIdx.x;
    const Dims& dm = P.dm;

    if (tid == 0) {
        for (int s = 0; s < P.ns; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), kConsumerWarps);  // every consumer warp releases
            sm.scnt[2 * s] = sm.scnt[2 * s + 1] = 0;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // Barrier count at launch: a multiple of nb plus arrivals of CTAs that already
        // reached this launch's first barrier (which cannot complete before we arrive).
        const uint64_t raw = ld_acquire_u64(ctl + kCtlBar);
        reinterpret_cast<unsigned long long*>(sm.flag)[1] = raw - raw % (uint64_t)P.nb;
        sm.flag[0] = read_status(ctl);
        if (blockIdx.x == 0) ctl[kCtlArgmax] = 0ull;  // step 0's argmax slot
    }
    __syncthreads();
    const uint64_t base = reinterpret_cast<unsigned long long*>(sm.flag)[1];
    if (sm.flag[0] != 0) return;  // an earlier launch failed: refuse until reset
    __syncthreads();

    if (tid >= kConsumerThreads) {  // producer warp
        if (tid == kConsumerThreads) {
            Producer pr(P, sm, ctl, base);
            pr.run();
        }
        return;
    }

    // ---------------- consumers
    int32_t* tokens_in = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(P.arena) + P.lay.tokens_in);
    float* xg = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.x);
    const __nv_bfloat16* embed = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.embed);
    long long epoch = 0;
    Ring rg;
    StepCtx sc;
    bool ok = true;
    Tracer tr;
    if (P.trace && tid == 0 && blockIdx.x % P.trace_every == 0) {
        tr.row0 = P.trace + (size_t)(blockIdx.x / P.trace_every) * P.trace_rows * kTraceWords;
        tr.rows = P.trace_rows;
        tr.mark(0);
    }
    const int own0 = (int)((long long)dm.d * blockIdx.x / P.nb);
    const int own1 = (int)((long long)dm.d * (blockIdx.x + 1) / P.nb);

    for (int t = 0; t < P.steps && ok; ++t) {
        sc.t = t;
        sc.p = P.pos0 + t;
        sc.lm_best = 0ull;
        if (tid == 0) {
            int tok;
            if (t < P.n_pending) {
                tok = __ldcg(tokens_in + t);
            } else {
                tok = key_index(__ldcg(ctl + kCtlArgmax + 16 * ((t - 1) % 3)));
                if (blockIdx.x == 0) P.tokens_out[t - P.n_pending] = tok;
            }
            if (blockIdx.x == 0) ctl[kCtlArgmax + 16 * ((t + 1) % 3)] = 0ull;
            sm.flag[2] = tok;
        }
        if (tid < dm.hd / 2) {
            const double freq = pow((double)dm.theta, -2.0 * (double)tid / (double)dm.hd);
            double s, c;
            sincos((double)sc.p * freq, &s, &c);
            sm.rope[tid] = make_float2((float)c, (float)s);
        }
        consumer_sync();
        const int tok = sm.flag[2];
        const __nv_bfloat16* erow = embed + (size_t)tok * dm.d;
        for (int i = own0 + tid; i < own1; i += kConsumerThreads) __stcg(xg + i, __bfloat162float(erow[i]));

        for (int l = 0; l < dm.L && ok; ++l) {
            sc.l = l;
            const uint8_t* lb = P.arena + P.lay.layer0 + (size_t)l * P.lay.layer_stride;
            const __nv_bfloat16* gattn = reinterpret_cast<const __nv_bfloat16*>(lb + P.lay.l_attn_norm);
            const __nv_bfloat16* gffn = reinterpret_cast<const __nv_bfloat16*>(lb + P.lay.l_ffn_norm);
            // attention block
            if (l == 0) load_rmsnorm(sm, nullptr, erow, gattn, dm.d, dm.eps);
            else load_rmsnorm(sm, xg, nullptr, gattn, dm.d, dm.eps);
            if (tid == 0) tr.mark(1);
            run_gemv(P, sm, ctl, kQKV, l, rg, sc, ok);
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
            if (tid == 0) tr.mark(1);
            if (dm.hd == 128) run_attention<128>(P, sm, ctl, l, rg, sc, ok);
            else run_attention<64>(P, sm, ctl, l, rg, sc, ok);
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
            load_vector(sm, reinterpret_cast<const float*>(P.arena + P.lay.o), dm.qd);
            if (tid == 0) tr.mark(1);
            run_gemv(P, sm, ctl, kO, l, rg, sc, ok);
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
            // feed-forward block
            load_rmsnorm(sm, xg, nullptr, gffn, dm.d, dm.eps);
            if (tid == 0) tr.mark(1);
            run_gemv(P, sm, ctl, kGU, l, rg, sc, ok);
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
            load_vector(sm, reinterpret_cast<const float*>(P.arena + P.lay.hdn), dm.F);
            if (tid == 0) tr.mark(1);
            run_gemv(P, sm, ctl, kD, l, rg, sc, ok);
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
        }
        if (!ok) break;
        if (step_has_head(P, t)) {
            load_rmsnorm(sm, xg, nullptr, reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.final_norm),
                         dm.d, dm.eps);
            if (tid == 0) tr.mark(1);
            run_gemv(P, sm, ctl, kLM, 0, rg, sc, ok);
            if ((tid & 31) == 0) sm.best[tid >> 5] = sc.lm_best;
            consumer_sync();
            if (tid == 0 && ok) {
                unsigned long long b = 0ull;
                for (int w = 0; w < kConsumerWarps; ++w) b = sm.best[w] > b ? sm.best[w] : b;
                atomicMax(ctl + kCtlArgmax + 16 * (t % 3), b);
            }
            if (!(ok = grid_sync(sm, epoch, base, P, ctl, ok, tr))) break;
        }
    }
    if (ok && blockIdx.x == 0 && tid == 0) {
        int32_t last;
        if (P.n_gen > 0) {
            last = key_index(__ldcg(ctl + kCtlArgmax + 16 * ((P.steps - 1) % 3)));
            P.tokens_out[P.n_gen - 1] = last;
        } else {
            last = __ldcg(tokens_in + P.n_pending - 1);
        }
        tokens_in[0] = last;  // pending input of the next call
    }
}

// ------------------------------------------------------------------ host-side launch

int monokernel_occupancy(int smem_bytes, int* blocks_per_sm) {
    cudaError_t e = cudaFuncSetAttribute(monokernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return (int)e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, monokernel, kThreads, smem_bytes);
    return (int)e;
}

void launch_decode(const Params& p, void* stream, int smem_bytes, int* err) {
    void* args[] = {const_cast<Params*>(&p)};
    cudaError_t e = cudaLaunchCooperativeKernel((const void*)monokernel, dim3(p.nb), dim3(kThreads), args,
                                                (size_t)smem_bytes, (cudaStream_t)stream);
    *err = (int)e;
}

}  // namespace kd
