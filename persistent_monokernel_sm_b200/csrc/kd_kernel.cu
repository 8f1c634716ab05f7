// kd_kernel.cu -- the decode monokernel: one persistent cooperative launch per kd_decode
// that runs every decode step of the request, layer after layer, without returning to the
// host ("3000 tokens per second: how to speed up LLMs on ordinary GPUs", aikraft.ru,
// section 04 "Monokernel and optimized GPU code": one resident GPU program covering matrix
// products, attention, normalisation and sampling, with tight control of synchronisation,
// prefetch and execution order).
//
// B200 design (one CTA per SM, 148 CTAs):
//  * Warp specialisation. Warp 7 of each CTA is the producer: one lane walks the CTA's
//    fixed schedule of weight tiles (and KV-cache tiles) and streams them HBM -> shared
//    memory with 1-D bulk async copies (cp.async.bulk) into a ring of 32 KB stages guarded
//    by mbarriers. Warps 0-6 are consumers; every consumer warp takes part in every stage
//    in order (a parity wait on an mbarrier can only tell the current phase from the one
//    before it, so a warp must have finished a slot's previous stage before it waits on
//    the slot again). 256 threads per CTA leave each thread the full 255 registers.
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
__device__ __forceinline__ unsigned int atom_add_acq_rel_u32(unsigned int* p, unsigned int v) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Tagged activation words: value (fp32 bits) in the low half, the producing phase's tag in
// the high half. A 64-bit store is single-copy atomic, so a reader that sees the tag sees
// the value written with it; no fence or barrier orders the two.
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, uint32_t tag) {
    const unsigned long long w = ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
// Two consecutive tagged words (16-byte aligned); each 8-byte element is read atomically.
__device__ __forceinline__ ulonglong2 ld_tagged2(const unsigned long long* p) {
    ulonglong2 w;
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w.x), "=l"(w.y) : "l"(p));
    return w;
}
__device__ __forceinline__ float tagged_value(unsigned long long w) { return __uint_as_float((uint32_t)w); }
__device__ __forceinline__ bool tagged_pair_is(const ulonglong2& w, uint32_t tag) {
    return (uint32_t)(w.x >> 32) == tag && (uint32_t)(w.y >> 32) == tag;
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
// The first error of a launch wins: its code goes to the status word, its place to kCtlWhere.
__device__ __noinline__ void raise_status(unsigned long long* ctl, int code, int where) {
    if (atomicCAS(ctl + kCtlStatus, 0ull, (unsigned long long)code) == 0ull)
        atomicExch(ctl + kCtlWhere, (unsigned long long)where);
}
__device__ __forceinline__ void raise_timeout(unsigned long long* ctl, int where) {
    raise_status(ctl, kStatusTimeout, where);
}

// Where a wait gave up or an input was refused: (what << 24) | (cta << 8) | detail.
enum { kWhereFull = 1, kWhereEmpty = 2, kWhereGrid = 3, kWhereKv = 4, kWhereToken = 5, kWhereData = 6 };
__device__ __forceinline__ int where_code(int what, int detail) {
    return (what << 24) | ((int)blockIdx.x << 8) | (detail & 0xff);
}

// Optional per-phase timestamps (SM cycles) of one CTA, recorded by consumer thread 0.
struct Tracer {
    unsigned long long* row0 = nullptr;
    int row = 0, rows = 0;
    unsigned long long waited = 0;  // cycles thread 0 spent on full-stage waits this phase
    __device__ void mark(int col) {
        if (row0 && row < rows - 1) row0[(size_t)row * kTraceWords + col] = (unsigned long long)clock64();
    }
    __device__ void next() {
        if (row0 && row < rows - 1) row0[(size_t)row * kTraceWords + 6] = waited;
        waited = 0;
        ++row;
    }
};

// 64-bit slots of the shared-memory flag words (sm.flag, 16 ints): the barrier counter base
// and the grid barriers done (thread 0 only); ints 0-3 are broadcast slots.
constexpr int kFlagBase = 4, kFlagEpoch = 5;
// Lane that performs a warp's shared-memory bookkeeping (see run_gemv).
constexpr int kSyncLane = 31;
static_assert(kGroupWarps == 8, "GEMV slice arithmetic assumes 8 warps per group");

// ------------------------------------------------------------------ schedule geometry
// Both the producer and the consumers enumerate the same stage sequence from these.

enum Phase { kQKV = 0, kATT = 1, kO = 2, kGU = 3, kD = 4, kLM = 5 };

struct Gemv {
    const uint8_t* base;  // matrix rows
    int K;                // reduction length (bf16 elements per row)
    int row0, row1;       // this CTA's rows
    int R;                // rows per stage
    int nst;              // stages
};

// log2 of the slices per row of a GEMV stage with R rows: 16 / R for R >= 2, 8 for R == 1
// (R is a power of two <= 8; see run_gemv_t).
__device__ __forceinline__ int gemv_log_slices(int R) {
    const int lr = __ffs(R) - 1;
    return R >= 2 ? 4 - lr : 3;
}

// This CTA's rows of every GEMV phase, [phase][row0, row1, stages], and the residual rows
// it owns: computed once per launch into shared memory (the 64-bit divisions that split the
// rows over the grid would otherwise be paid by every warp at every phase).
constexpr int kGeomOwn = 18, kGeomWords = 32;
__device__ void cta_geometry(const Params& P, int c, int* geom) {
    const Dims& dm = P.dm;
    for (int phase = 0; phase < 6; ++phase) {
        int units = 0, rpu = 1, R = 1;
        switch (phase) {
            case kQKV: units = dm.qkv_rows / 2; rpu = 2; R = P.rows_qkv; break;
            case kO: units = dm.d; R = P.rows_o; break;
            case kGU: units = dm.F; rpu = 2; R = P.rows_gu; break;  // (gate, up) row pairs
            case kD: units = dm.d; R = P.rows_d; break;
            case kLM: units = dm.V; R = P.rows_lm; break;
            default: break;
        }
        const int row0 = (int)((long long)units * c / P.nb) * rpu;
        const int row1 = (int)((long long)units * (c + 1) / P.nb) * rpu;
        geom[3 * phase] = row0;
        geom[3 * phase + 1] = row1;
        geom[3 * phase + 2] = (row1 - row0 + R - 1) / R;
    }
    geom[kGeomOwn] = (int)((long long)dm.d * c / P.nb);
    geom[kGeomOwn + 1] = (int)((long long)dm.d * (c + 1) / P.nb);
}

__device__ __forceinline__ Gemv gemv_geom(const Params& P, const int* geom, int phase, int l) {
    const Dims& dm = P.dm;
    const uint8_t* lb = P.arena + P.lay.layer0 + (size_t)l * P.lay.layer_stride;
    Gemv g;
    switch (phase) {
        case kQKV: g.base = lb + P.lay.l_wqkv; g.K = dm.d; g.R = P.rows_qkv; break;
        case kO: g.base = lb + P.lay.l_wo; g.K = dm.qd; g.R = P.rows_o; break;
        case kGU: g.base = lb + P.lay.l_wgu; g.K = dm.d; g.R = P.rows_gu; break;
        case kD: g.base = lb + P.lay.l_wd; g.K = dm.F; g.R = P.rows_d; break;
        default: g.base = P.arena + P.lay.lm_head; g.K = dm.d; g.R = P.rows_lm; break;
    }
    g.row0 = geom[3 * phase];
    g.row1 = geom[3 * phase + 1];
    g.nst = geom[3 * phase + 2];
    return g;
}

struct Attn {
    int g, piece;  // kv head, piece index (g < 0: this CTA has no piece)
    int a, b;      // positions [a, b) of the piece (b may include the current position)
    int tma_end;   // [a, tma_end) streamed through the ring; position p handled directly
    int nst;       // ring stages of the piece
};

constexpr int kLastPieceRelief = 64;
__device__ __forceinline__ Attn attn_geom(const Params& P, int p, int c) {
    Attn at;
    const int A = P.attn_pieces;
    if (c >= A * P.dm.Hkv) {
        at.g = -1;
        at.piece = 0;
        at.a = at.b = at.tma_end = at.nst = 0;
        return at;
    }
    at.g = c / A;
    at.piece = c % A;
    // The last piece also appends the current position, folds it in and usually combines the
    // head's pieces, so it takes kLastPieceRelief fewer cached positions than an even share;
    // the other pieces split the rest evenly.
    const long long T = (long long)p + 1;
    long long last = T / A - kLastPieceRelief;
    if (last < 1 || A == 1) last = A == 1 ? T : 1;
    if (at.piece == A - 1) {
        at.a = (int)(T - last);
        at.b = (int)T;
    } else {
        at.a = (int)((T - last) * at.piece / (A - 1));
        at.b = (int)((T - last) * (at.piece + 1) / (A - 1));
    }
    at.tma_end = at.b < p ? at.b : p;
    if (at.tma_end < at.a) at.tma_end = at.a;
    at.nst = (at.tma_end - at.a + P.pos_per_stage - 1) / P.pos_per_stage;
    return at;
}

// The LM head runs at steps that pick a token, or at every step when logits are dumped.
__device__ __forceinline__ bool step_has_head(const Params& P, int t) {
    return P.dump || t >= P.n_pending - 1;
}
// Phases run before step s begins (5 per layer, plus the LM head at steps that have one).
__device__ __forceinline__ long long phases_before_step(const Params& P, int s) {
    long long heads = P.dump ? s : (s - (P.n_pending - 1) > 0 ? s - (P.n_pending - 1) : 0);
    return (long long)s * 5 * P.dm.L + heads;
}
// Tag of phase q of step t (q = 5 * layer + phase, or 5 * L for the LM head). Every
// activation element a phase writes for other CTAs carries its tag in the same 64-bit word
// as the value, so a reader polls the data itself instead of a grid barrier.
__device__ __forceinline__ uint32_t phase_tag(const Params& P, int t, int q) {
    return P.tag0 + 1u + (uint32_t)(phases_before_step(P, t) + q);
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
    float* xown;            // the residual rows this CTA owns (updated by O and D)
    __nv_bfloat16* kvcur;   // the current position's K and V row of the head being attended
    int* geom;              // this CTA's GEMV rows per phase and owned residual rows (cta_geometry)
    Attn* att;              // this step's attention piece (consumers)
};

// Byte offsets of the shared-memory regions; each starts on a 128-byte boundary (vector
// loads and bulk-copy destinations need 16). Used by the kernel and for the launch size.
struct SmemLayout {
    size_t ring, xs, qs, rope, red, best, flag, full, empty, xown, kvcur, geom, att, total;
};
__host__ __device__ inline SmemLayout smem_layout(int ns, int xs_floats, int xown_floats) {
    SmemLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = (off + bytes + 127) & ~(size_t)127;
        return at;
    };
    L.ring = take((size_t)ns * kStageBytes);
    L.xs = take((size_t)xs_floats * 4);
    L.qs = take((size_t)kMaxGroup * 128 * 4);
    L.rope = take(64 * 8);
    L.red = take(64 * 4);
    L.best = take((size_t)kConsumerWarps * 8);
    L.flag = take(16 * 4);
    L.full = take((size_t)kMaxStages * 8);
    L.empty = take((size_t)kMaxStages * 8);
    L.xown = take((size_t)xown_floats * 4);
    L.kvcur = take(2 * 128 * 2);
    L.geom = take((size_t)kGeomWords * 4);
    L.att = take(sizeof(Attn));
    L.total = off;
    return L;
}

__device__ __forceinline__ Smem carve(const Params& P, uint8_t* base) {
    const SmemLayout L = smem_layout(P.ns, P.xs_floats, P.xown_floats);
    Smem s;
    s.ring = base + L.ring;
    s.xs = reinterpret_cast<float*>(base + L.xs);
    s.qs = reinterpret_cast<float*>(base + L.qs);
    s.rope = reinterpret_cast<float2*>(base + L.rope);
    s.red = reinterpret_cast<float*>(base + L.red);
    s.best = reinterpret_cast<unsigned long long*>(base + L.best);
    s.flag = reinterpret_cast<int*>(base + L.flag);
    s.full = reinterpret_cast<uint64_t*>(base + L.full);
    s.empty = reinterpret_cast<uint64_t*>(base + L.empty);
    s.xown = reinterpret_cast<float*>(base + L.xown);
    s.kvcur = reinterpret_cast<__nv_bfloat16*>(base + L.kvcur);
    s.geom = reinterpret_cast<int*>(base + L.geom);
    s.att = reinterpret_cast<Attn*>(base + L.att);
    return s;
}

int monokernel_smem_bytes(const Params& p) { return (int)smem_layout(p.ns, p.xs_floats, p.xown_floats).total; }

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

// `waited` accumulates the cycles spent here (read by the trace only).
__device__ __forceinline__ bool wait_full(const Smem& sm, const Ring& rg, const Params& P, unsigned long long* ctl,
                                          unsigned long long& waited) {
    const uint32_t a = smem_u32(&sm.full[rg.slot]);
    if (__all_sync(0xffffffffu, mbar_try_wait(a, rg.phase))) return true;
    const long long c0 = clock64();
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (__all_sync(0xffffffffu, mbar_wait_hint(a, rg.phase))) {
            waited += (unsigned long long)(clock64() - c0);
            return true;
        }
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

// End of a phase inside a step: every consumer warp is done with xs, and the CTA agrees on
// whether every wait succeeded (a failed CTA stops; the others stop at their next wait, which
// sees the status word).
__device__ __forceinline__ bool phase_end(bool local_ok, Tracer& tr) {
    const bool cta_ok = consumer_sync_and(local_ok);
    if (threadIdx.x == 0) {
        tr.mark(2);
        tr.mark(3);
        tr.next();
        tr.mark(0);
    }
    return cta_ok;
}

// Re-read a 16-byte pair of tagged words until both carry `tag` (the first read was issued
// by the caller together with its other loads). Gives up, with the device status set, when
// another wait has failed or after the time limit; `what` identifies the buffer.
// Returns the pair; its tags differ from `tag` only when the wait gave up.
__device__ __noinline__ ulonglong2 poll_pair(const unsigned long long* p, uint32_t tag, const Params& P,
                                             unsigned long long* ctl, int what) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        const ulonglong2 w = ld_tagged2(p);
        if (tagged_pair_is(w, tag)) return w;
        if ((it & 31) == 0) {
            if (read_status(ctl) != 0) return w;
            if (globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                raise_timeout(ctl, where_code(kWhereData, what));
                return w;
            }
        }
    }
}
__device__ __forceinline__ bool get_pair(const unsigned long long* p, uint32_t tag, ulonglong2& w, const Params& P,
                                         unsigned long long* ctl, int what) {
    if (tagged_pair_is(w, tag)) return true;
    w = poll_pair(p, tag, P, ctl, what);
    return tagged_pair_is(w, tag);
}

// Grid-wide barrier among the consumer warps of all CTAs. `epoch` counts barriers this
// launch has completed; arrivals accumulate in one monotonic counter, so there is no
// reset race and a barrier completes when the counter reaches base + epoch * nb.
// `local_ok` is false in a warp whose wait gave up; the result is the same for every
// consumer thread of the CTA, and false in every CTA once any wait anywhere has given up
// (the device status word is re-read after the barrier completes).
// The counter base of this launch and the barriers done so far live in shared memory
// (kFlagBase, kFlagEpoch): only thread 0 uses them, so no thread carries them in registers.
__device__ __forceinline__ bool grid_sync(const Smem& sm, const Params& P, unsigned long long* ctl, bool local_ok,
                                          Tracer& tr) {
    // every consumer warp's writes of this phase are done; did every warp succeed?
    const bool cta_ok = consumer_sync_and(local_ok);
    if (threadIdx.x == 0) tr.mark(2);
    if (threadIdx.x == 0 && !cta_ok) sm.flag[0] = 0;
    if (threadIdx.x == 0 && cta_ok) {
        // The release add publishes every consumer thread's writes of this phase (ordered
        // before it by the CTA barrier above); the acquire poll below makes all CTAs'
        // writes visible to this thread, and the CTA barrier after it to the others. Loads
        // of data written during the launch bypass L1 (ld.global.cg), so no fence is needed.
        red_release_add_u64(ctl + kCtlBar, 1ull);
        unsigned long long* bs = reinterpret_cast<unsigned long long*>(sm.flag);
        const long long epoch = (long long)bs[kFlagEpoch];
        bs[kFlagEpoch] = (unsigned long long)(epoch + 1);
        const uint64_t target = bs[kFlagBase] + (uint64_t)(epoch + 1) * (uint64_t)P.nb;
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
        if (ok && read_status(ctl) != 0) ok = 0;
        sm.flag[0] = ok;
        tr.mark(3);
        tr.next();
        tr.mark(0);
    }
    consumer_sync();
    return sm.flag[0] != 0;
}

// ------------------------------------------------------------------ activation loads

// Shared-memory store in asm: the compiler then does not treat it as a possible write to a
// global source, and may keep later iterations' global loads ahead of it (the asm stays
// ordered with the barriers, also volatile asm).
__device__ __forceinline__ void sts128(float* p, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w));
}

// Tagged vectors are read two float4 groups (four 16-byte loads) per thread at a time, all
// four loads issued before any tag is checked, so a pair of groups whose data is ready costs
// one L2 round trip; a stale pair is re-polled until it carries `tag` (`ok` turns false if
// that wait gives up). The loads go to named registers: arrays written by asm get a stack
// slot.
struct Tagged2x4 {
    ulonglong2 a0, b0, a1, b1;
};
__device__ __forceinline__ void load_groups(const unsigned long long* src, int k0, int k1, bool h1, Tagged2x4& t) {
    t.a0 = ld_tagged2(src + k0);
    t.b0 = ld_tagged2(src + k0 + 2);
    if (h1) {
        t.a1 = ld_tagged2(src + k1);
        t.b1 = ld_tagged2(src + k1 + 2);
    }
}
__device__ __forceinline__ float4 group_value(const unsigned long long* src, int k, uint32_t tag, ulonglong2 a, ulonglong2 b,
                                              const Params& P, unsigned long long* ctl, int what, bool& ok) {
    if (!get_pair(src + k, tag, a, P, ctl, what) || !get_pair(src + k + 2, tag, b, P, ctl, what)) ok = false;
    return make_float4(tagged_value(a.x), tagged_value(a.y), tagged_value(b.x), tagged_value(b.y));
}

// xs <- x * rsqrt(mean(x^2) + eps) * g in split layout. src_ll: a tagged vector written
// during the launch by the phase with tag `tag`; else src_bf16, an embedding row.
__device__ __forceinline__ void load_rmsnorm(const Smem& sm, const unsigned long long* src_ll, uint32_t tag,
                                             const __nv_bfloat16* src_bf16, const __nv_bfloat16* gain, int K, float eps,
                                             const Params& P, unsigned long long* ctl, bool& ok) {
    const int tid = threadIdx.x;
    constexpr int step = kConsumerThreads * 4;
    // With K <= 2 * step (every model up to d_model 2048) each thread's gains are read here,
    // before the input is polled, so the normalisation below waits on no global load.
    const bool early = K <= 2 * step;
    uint2 g0 = make_uint2(0u, 0u), g1 = make_uint2(0u, 0u);
    if (early) {
        if (tid * 4 < K) g0 = __ldg(reinterpret_cast<const uint2*>(gain + tid * 4));
        if (tid * 4 + step < K) g1 = __ldg(reinterpret_cast<const uint2*>(gain + tid * 4 + step));
    }
    float ss = 0.f;
    for (int k0 = tid * 4; k0 < K; k0 += 2 * step) {
        const int k1 = k0 + step;
        const bool h1 = k1 < K;
        float4 v0, v1;
        if (src_ll) {
            Tagged2x4 t;
            load_groups(src_ll, k0, k1, h1, t);
            v0 = group_value(src_ll, k0, tag, t.a0, t.b0, P, ctl, 1, ok);
            if (h1) v1 = group_value(src_ll, k1, tag, t.a1, t.b1, P, ctl, 1, ok);
        } else {
            const uint2 e0 = __ldg(reinterpret_cast<const uint2*>(src_bf16 + k0));
            const uint2 e1 = h1 ? __ldg(reinterpret_cast<const uint2*>(src_bf16 + k1)) : make_uint2(0, 0);
            v0 = make_float4(bf_lo(e0.x), bf_hi(e0.x), bf_lo(e0.y), bf_hi(e0.y));
            v1 = make_float4(bf_lo(e1.x), bf_hi(e1.x), bf_lo(e1.y), bf_hi(e1.y));
        }
        ss += v0.x * v0.x + v0.y * v0.y + v0.z * v0.z + v0.w * v0.w;
        sts128(&sm.xs[xs_index(k0, K)], v0);
        if (h1) {
            ss += v1.x * v1.x + v1.y * v1.y + v1.z * v1.z + v1.w * v1.w;
            sts128(&sm.xs[xs_index(k1, K)], v1);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) sm.red[tid >> 5] = ss;
    consumer_sync();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += sm.red[w];
    const float inv = 1.0f / sqrtf(tot / (float)K + eps);
    for (int k = tid * 4; k < K; k += step) {
        float4* p = reinterpret_cast<float4*>(&sm.xs[xs_index(k, K)]);
        const uint2 gw = early ? (k == tid * 4 ? g0 : g1) : __ldg(reinterpret_cast<const uint2*>(gain + k));
        float4 v = *p;
        v.x = (v.x * inv) * bf_lo(gw.x);
        v.y = (v.y * inv) * bf_hi(gw.x);
        v.z = (v.z * inv) * bf_lo(gw.y);
        v.w = (v.w * inv) * bf_hi(gw.y);
        *p = v;
    }
    consumer_sync();
}

// xs <- a tagged vector written during the launch by the phase with tag `tag`.
__device__ __forceinline__ void load_vector(const Smem& sm, const unsigned long long* src, uint32_t tag, int K,
                                            const Params& P, unsigned long long* ctl, bool& ok) {
    constexpr int step = kConsumerThreads * 4;
    for (int k0 = threadIdx.x * 4; k0 < K; k0 += 2 * step) {
        const int k1 = k0 + step;
        const bool h1 = k1 < K;
        Tagged2x4 t;
        load_groups(src, k0, k1, h1, t);
        sts128(&sm.xs[xs_index(k0, K)], group_value(src, k0, tag, t.a0, t.b0, P, ctl, 2, ok));
        if (h1) sts128(&sm.xs[xs_index(k1, K)], group_value(src, k1, tag, t.a1, t.b1, P, ctl, 2, ok));
    }
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
    uint32_t tag;                // tag of the phase being run (its outputs carry it)
    unsigned long long lm_best;  // running argmax key of this warp (lane 0)
};

// Output of one finished GEMV row (global row index `row`, value y), tagged with the phase:
// stored raw for the Q/K/V projections (RoPE and the KV-cache append are applied where
// they are consumed), the FFN hidden value silu(gate) * up for a gate/up pair (y is already
// that value; `row` is the pair's index), added into the residual for O and down (the CTA
// owns those rows and keeps them in shared memory, so no read-back from L2; O's results go
// to x copy 0, D's to copy 1), and for the LM head dumped when requested and folded into
// this thread's running argmax.
__device__ __forceinline__ void row_out(const Params& P, const Smem& sm, int phase, int row, float y, StepCtx& sc,
                                        int own0) {
    unsigned long long* arena = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena));
    if (phase == kQKV) {
        st_tagged(arena + P.lay.qkv / 8 + row, y, sc.tag);
    } else if (phase == kGU) {
        st_tagged(arena + P.lay.gu / 8 + row, y, sc.tag);  // `row`: the pair (hidden unit) index
    } else if (phase == kO || phase == kD) {
        const float v = sm.xown[row - own0] + y;
        sm.xown[row - own0] = v;
        st_tagged(arena + P.lay.x / 8 + (phase == kO ? 0 : P.dm.d) + row, v, sc.tag);
    } else {
        if (P.dump) __stcg(P.logits_out + (size_t)sc.t * P.dm.V + row, y);
        const unsigned long long key = argmax_key(y, row);
        if (key > sc.lm_best) sc.lm_best = key;
    }
}

// One GEMV phase. A stage holds R rows (R a power of two <= 8); each row is cut into KS
// slices of the reduction dimension and the 8 warps share the R * KS (row, slice) units:
//   R >= 2: KS = 16 / R, 16 units, warp w takes units w and w + 8 -- the same slice of two
//           rows R / 2 apart, so one activation slice in registers serves both;
//   R == 1: KS = 8, warp w takes slice w of the one row.
// The slice is at most 1024 elements when R >= 2 (4 chunks of 8 per lane), which keeps the
// kernel's register demand low enough to avoid spilling. A warp's slice sums go to xs (free
// once every warp holds its activation slice) as [local row][slice]; after the last stage
// the rows are summed in slice order and put out (row_out), the gate/up rows in pairs.
// NCL > 0: every slice is exactly NCL chunks per lane, so the chunk loop has no bounds test.
// A wait that gives up marks `ok` false and the warp skips the work of the remaining stages,
// but it still reaches every named barrier; the phase end then reports the failure to the
// whole CTA at once.
template <int NCL, int MAXCH>
__device__ __forceinline__ void run_gemv_t(const Params& P, const Smem& sm_ref, unsigned long long* ctl, int phase, int l,
                                        Ring& rg_ref, StepCtx& sc_ref, bool& ok_ref, Tracer& tr) {
    const Smem sm = sm_ref;
    Ring rg = rg_ref;
    StepCtx sc = sc_ref;
    bool ok = ok_ref;
    const Gemv g = gemv_geom(P, sm.geom, phase, l);
    const int nst = g.nst;
    const int ns = P.ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool dual = g.R >= 2;
    const int lks = gemv_log_slices(g.R), KS = 1 << lks;  // slices per row
    const int ks = warp & (KS - 1);                        // this warp's slice
    const int rowa = warp >> lks, rowb = (warp + 8) >> lks;  // its rows within a stage
    const int nch = g.K >> 3;
    const int c0 = (nch * ks) >> lks, c1 = (nch * (ks + 1)) >> lks;  // at most 32 * kMaxChunks chunks
    const size_t rowbytes = (size_t)g.K * 2;
    const int own0 = sm.geom[kGeomOwn];
    unsigned long long& waited = tr.waited;

    // this lane's activation chunks: c = c0 + lane + 32 i
    constexpr int NX = NCL > 0 ? NCL : MAXCH;
    float xr[NX][8];
    const float4* xlo = reinterpret_cast<const float4*>(sm.xs);
    const float4* xhi = reinterpret_cast<const float4*>(sm.xs + (g.K >> 1));
#pragma unroll
    for (int i = 0; i < NX; ++i) {
        const int c = c0 + lane + 32 * i;
        const bool in = NCL > 0 || c < c1;
        const float4 a = in ? xlo[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 b = in ? xhi[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        xr[i][0] = a.x, xr[i][1] = a.y, xr[i][2] = a.z, xr[i][3] = a.w;
        xr[i][4] = b.x, xr[i][5] = b.y, xr[i][6] = b.z, xr[i][7] = b.w;
    }
    if (threadIdx.x == 0) tr.mark(7);  // activation slice in registers
    float* pp = sm.xs;
    consumer_sync();  // every warp has its slice: xs now takes the slice sums

    auto dot_row = [&](const uint8_t* wrow) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const uint8_t* wl = wrow + (c0 + lane) * 16;  // this lane's first chunk; then +512 B each
#pragma unroll
        for (int i = 0; i < NX; ++i) {
            if (NCL > 0 || c0 + lane + 32 * i < c1) {
                const uint4 w = *reinterpret_cast<const uint4*>(wl + i * 512);
                a0 = fmaf(bf_lo(w.x), xr[i][0], a0);
                a1 = fmaf(bf_hi(w.x), xr[i][1], a1);
                a2 = fmaf(bf_lo(w.y), xr[i][2], a2);
                a3 = fmaf(bf_hi(w.y), xr[i][3], a3);
                a0 = fmaf(bf_lo(w.z), xr[i][4], a0);
                a1 = fmaf(bf_hi(w.z), xr[i][5], a1);
                a2 = fmaf(bf_lo(w.w), xr[i][6], a2);
                a3 = fmaf(bf_hi(w.w), xr[i][7], a3);
            }
        }
        return (a0 + a1) + (a2 + a3);
    };

    // Stages are taken four at a time, as two pairs. For each pair the four dot products (two
    // rows of each stage) are formed and both slots handed back; the eight lane partials of
    // the four stages are then reduced together. Three exchange levels (offsets 16, 8, 4) halve
    // the values a lane holds at each step, so 4 + 2 + 1 shuffles leave each lane one value
    // summed over 8 lanes; two plain levels (offsets 2, 1) complete the 32-lane sum. Value i
    // (stage j + i / 2, row a for even i, row b for odd i) ends in lanes 4i..4i+3.
    auto put = [&](int jj, int row, float z) {
        if (jj < nst && row < min(g.R, g.row1 - (g.row0 + jj * g.R))) pp[(jj * g.R + row) * KS + ks] = z;
    };
    for (int j = 0; j < nst; j += 4) {
        float v[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // stages j + 2h and j + 2h + 1
            const int jj = j + 2 * h;
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
            if (jj < nst) {
                const Ring ra = rg;
                rg.advance(ns);
                const bool two = jj + 1 < nst;
                const Ring rb = rg;
                if (two) rg.advance(ns);
                if (ok) {
                    if (!wait_full(sm, ra, P, ctl, waited) || (two && !wait_full(sm, rb, P, ctl, waited))) {
                        ok = false;
                    } else {
                        if (threadIdx.x == 0 && jj == 0) tr.mark(4);  // first stage of the phase ready
                        const int na = min(g.R, g.row1 - (g.row0 + jj * g.R));                   // rows in stage jj
                        const int nb = two ? min(g.R, g.row1 - (g.row0 + (jj + 1) * g.R)) : 0;  // and in jj + 1
                        const uint8_t* sa = sm.ring + (size_t)ra.slot * kStageBytes;
                        const uint8_t* sb = sm.ring + (size_t)rb.slot * kStageBytes;
                        p0 = rowa < na ? dot_row(sa + rowa * rowbytes) : 0.f;
                        p1 = dual && rowb < na ? dot_row(sa + rowb * rowbytes) : 0.f;
                        p2 = rowa < nb ? dot_row(sb + rowa * rowbytes) : 0.f;
                        p3 = dual && rowb < nb ? dot_row(sb + rowb * rowbytes) : 0.f;
                        __syncwarp();
                        if (lane == kSyncLane) {  // done with the stages
                            mbar_arrive(smem_u32(&sm.empty[ra.slot]));
                            if (two) mbar_arrive(smem_u32(&sm.empty[rb.slot]));
                        }
                    }
                }
            }
            v[4 * h] = p0, v[4 * h + 1] = p1, v[4 * h + 2] = p2, v[4 * h + 3] = p3;
        }
        const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
        float w4[4], w2[2];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w4[k] = (b4 ? v[4 + k] : v[k]) + __shfl_xor_sync(0xffffffffu, b4 ? v[k] : v[4 + k], 16);
#pragma unroll
        for (int k = 0; k < 2; ++k)
            w2[k] = (b3 ? w4[2 + k] : w4[k]) + __shfl_xor_sync(0xffffffffu, b3 ? w4[k] : w4[2 + k], 8);
        float z = (b2 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? w2[0] : w2[1], 4);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        if ((lane & 3) == 0 && ok) {
            const int i = lane >> 2;  // value index: 4 * b4 + 2 * b3 + b2
            if ((i & 1) == 0) put(j + (i >> 1), rowa, z);
            else if (dual) put(j + (i >> 1), rowb, z);
        }
    }
    if (threadIdx.x == 0) tr.mark(5);  // this warp's stages done
    consumer_sync();
    const int nrows = g.row1 - g.row0;
    for (int i = threadIdx.x; i < nrows; i += kConsumerThreads) {
        float tot = 0.f;
        for (int q = 0; q < KS; ++q) tot += pp[i * KS + q];
        if (phase != kGU) {
            row_out(P, sm, phase, g.row0 + i, tot, sc, own0);
        } else if ((i & 1) == 0) {
            // interleaved (gate, up) rows: the FFN hidden value silu(gate) * up
            float up = 0.f;
            for (int q = 0; q < KS; ++q) up += pp[(i + 1) * KS + q];
            row_out(P, sm, phase, (g.row0 + i) >> 1, tot / (1.0f + expf(-tot)) * up, sc, own0);
        }
    }
    rg_ref = rg;
    ok_ref = ok;
    // LM head: fold the lanes' running argmax into lane 0's (lowest index on ties)
    if (phase == kLM) {
        unsigned long long key = sc.lm_best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
            key = other > key ? other : key;
        }
        sc_ref.lm_best = key;
    }
}

// Chunks (8 elements) per lane of every warp's slice when that count is exact, else 0.
__device__ __forceinline__ int gemv_exact_chunks(int K, int R) {
    const int lks = gemv_log_slices(R);
    const int nch = K >> 3, per = nch >> (5 + lks);
    return (per << (5 + lks)) == nch && per <= kMaxChunks ? per : 0;
}

// MAXCH (4 or 8): the most chunks per lane any phase of this model needs; the kernel is
// instantiated per MAXCH so that a model whose slices fit in 4 chunks never carries the
// registers of an 8-chunk loop.
template <int MAXCH>
__device__ __forceinline__ void run_gemv(const Params& P, const Smem& sm, unsigned long long* ctl, int phase, int l,
                                         Ring& rg, StepCtx& sc, bool& ok, Tracer& tr) {
    const Gemv g = gemv_geom(P, sm.geom, phase, l);
    switch (gemv_exact_chunks(g.K, g.R)) {
        case 1: run_gemv_t<1, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 2: run_gemv_t<2, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 3: run_gemv_t<3, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 4: run_gemv_t<4, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 5: if constexpr (MAXCH >= 5) run_gemv_t<5, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 6: if constexpr (MAXCH >= 6) run_gemv_t<6, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 7: if constexpr (MAXCH >= 7) run_gemv_t<7, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        case 8: if constexpr (MAXCH >= 8) run_gemv_t<8, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
        default: run_gemv_t<0, MAXCH>(P, sm, ctl, phase, l, rg, sc, ok, tr); break;
    }
}

// Loads of K and V rows from a stage of the shared-memory ring.
__device__ __forceinline__ uint4 ld16(const __nv_bfloat16* p) { return *reinterpret_cast<const uint4*>(p); }
template <int E>
__device__ __forceinline__ void ld_v(const __nv_bfloat16* p, float (&v)[E]) {
    if constexpr (E == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        v[0] = bf_lo(w.x), v[1] = bf_hi(w.x), v[2] = bf_lo(w.y), v[3] = bf_hi(w.y);
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        v[0] = bf_lo(w), v[1] = bf_hi(w);
    }
}

// Split-K decode attention for one kv head over this CTA's piece of the cache. Each warp
// handles 8 positions per pass: lanes 4j..4j+3 hold position j's score (each lane a quarter
// of the head dimension, q broadcast from shared memory), one max / rescale per pass, then
// all lanes accumulate the 8 V rows (each lane hd/32 output dims). States of the warps are
// merged per CTA; the last CTA of a kv head to finish combines all pieces.
// GMAX >= the number of q heads per kv head (2, 4 or 8).
constexpr int kCombineBatch = 18;  // pieces whose records one combining thread loads at once
template <int HD, int GMAX>
__device__ __forceinline__ void run_attention(const Params& P, const Smem& sm_ref, unsigned long long* ctl, int l,
                                          Ring& rg_ref, StepCtx& sc_ref, bool& ok_ref, Tracer& tr) {
    const Smem sm = sm_ref;
    const StepCtx sc = sc_ref;
    Ring rg = rg_ref;
    bool ok = ok_ref;
    constexpr int CPL = HD / 32;  // 16-byte K chunks per lane (4 lanes per position)
    constexpr int E = HD / 32;    // output dims per lane
    const Dims& dm = P.dm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int pj = lane >> 2, qq = lane & 3;
    const Attn at = *sm.att;  // this step's piece, set at the step start
    if (at.g < 0) return;  // uniform across the CTA
    const int r = dm.r, A = P.attn_pieces;
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
    // The Q/K/V projections arrive raw, q and k rows in RoPE-pair order (row 2i = dim i,
    // row 2i + 1 = dim i + hd/2). Rotate this group's q heads at position p while loading.
    // The piece that holds position p also appends that position's K (rotated) and V to the
    // cache, rounded to bf16, and keeps a copy for its own pass below. Every load of this
    // prologue is issued before any store (one L2 round trip): at most 2 q pairs per thread
    // (r * HD / 2 <= 512), and one K and one V pair for threads below HD / 2.
    // The projections are tagged words written by the QKV phase (tag one below this phase's).
    const unsigned long long* raw = reinterpret_cast<const unsigned long long*>(P.arena + P.lay.qkv);
    const uint32_t qkv_tag = sc.tag - 1u;
    const unsigned long long* qg = raw + (size_t)at.g * r * HD;
    const bool has_current = at.b > sc.p;
    const bool kv_lane = has_current && tid < HD / 2;
    float2 qv[2], kv2, vv2;
    {
        ulonglong2 wq[2], wk, wv;
        const unsigned long long* pq[2];
        const unsigned long long* pk = raw + dm.qd + (size_t)at.g * HD + 2 * tid;
        const unsigned long long* pv = pk + dm.kvd;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int t = tid + u * kConsumerThreads;
            pq[u] = qg + (t / (HD / 2)) * HD + 2 * (t % (HD / 2));
            if (t < r * HD / 2) wq[u] = ld_tagged2(pq[u]);
        }
        if (kv_lane) {
            wk = ld_tagged2(pk);
            wv = ld_tagged2(pv);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (tid + u * kConsumerThreads < r * HD / 2) {
                if (!get_pair(pq[u], qkv_tag, wq[u], P, ctl, 3)) ok = false;
                qv[u] = make_float2(tagged_value(wq[u].x), tagged_value(wq[u].y));
            }
        }
        if (kv_lane) {
            if (!get_pair(pk, qkv_tag, wk, P, ctl, 4) || !get_pair(pv, qkv_tag, wv, P, ctl, 4)) ok = false;
            kv2 = make_float2(tagged_value(wk.x), tagged_value(wk.y));
            vv2 = make_float2(tagged_value(wv.x), tagged_value(wv.y));
        }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int t = tid + u * kConsumerThreads;
        if (t < r * HD / 2) {
            const int hh = t / (HD / 2), i = t % (HD / 2);
            const float2 cs = sm.rope[i];
            sm.qs[hh * HD + i] = (qv[u].x * cs.x - qv[u].y * cs.y) * qscale;
            sm.qs[hh * HD + i + HD / 2] = (qv[u].y * cs.x + qv[u].x * cs.y) * qscale;
        }
    }
    if (kv_lane) {
        const int i = tid;
        const size_t off = (((size_t)l * dm.Hkv + at.g) * dm.S + sc.p) * HD;
        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.kcache) + off;
        __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.vcache) + off;
        const float2 cs = sm.rope[i];
        const __nv_bfloat16 k0 = __float2bfloat16_rn(kv2.x * cs.x - kv2.y * cs.y);
        const __nv_bfloat16 k1 = __float2bfloat16_rn(kv2.y * cs.x + kv2.x * cs.y);
        kc[i] = k0, kc[i + HD / 2] = k1;
        sm.kvcur[i] = k0, sm.kvcur[i + HD / 2] = k1;
        const __nv_bfloat162 v01 = __floats2bfloat162_rn(vv2.x, vv2.y);
        *reinterpret_cast<__nv_bfloat162*>(vc + 2 * i) = v01;
        *reinterpret_cast<__nv_bfloat162*>(&sm.kvcur[HD + 2 * i]) = v01;
    }
    // (Bulk copies read these rows at later steps only, after the step's grid barrier; the
    // producer issues the proxy fence after acquiring that barrier.)
    consumer_sync();
    if (tid == 0) tr.mark(4);

    // The current position's state is one record next to the warps' (slot kConsumerWarps of
    // the merge area): score s = q . k_cur, weight sum 1, accumulator v_cur. One warp forms it
    // before the pass over the cache, instead of a whole extra pass at the end.
    const int rec = HD + 2;
    float* ws = sm.xs;  // [warp][h][rec] merge area (xs is free during attention)
    if (has_current && warp == kConsumerWarps - 1) {
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h < r) {
                float sdot = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e)
                    sdot = fmaf(sm.qs[h * HD + lane * E + e], __bfloat162float(sm.kvcur[lane * E + e]), sdot);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
                float* wr = ws + ((size_t)kConsumerWarps * r + h) * rec;
                if (lane == 0) wr[0] = sdot, wr[1] = 1.f;
#pragma unroll
                for (int e = 0; e < E; ++e) wr[2 + lane * E + e] = __bfloat162float(sm.kvcur[HD + lane * E + e]);
            }
        }
    }

    float m[GMAX], lsum[GMAX], acc[GMAX][E];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        m[h] = -INFINITY;
        lsum[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
    }
    // One pass over two blocks of up to 8 positions each (A: rows at ka / va, B: rows at
    // kb / vb): lanes 4j..4j+3 score position j of both blocks, then all lanes fold the up
    // to 16 V rows into their output dims with a single rescale.
    auto pass2 = [&](const __nv_bfloat16* ka, const __nv_bfloat16* va, int na, const __nv_bfloat16* kb,
                     const __nv_bfloat16* vb, int nb) {
        const bool ma = pj < na, mb = pj < nb;
        float sa[GMAX][2], sb[GMAX][2];
#pragma unroll
        for (int h = 0; h < GMAX; ++h) sa[h][0] = sa[h][1] = sb[h][0] = sb[h][1] = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = qq + 4 * i;
            const uint4 wa = ma ? ld16(ka + (size_t)pj * HD + c * 8) : make_uint4(0, 0, 0, 0);
            const uint4 wb = mb ? ld16(kb + (size_t)pj * HD + c * 8) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                if (h < r) {
                    const float4 qa = *reinterpret_cast<const float4*>(&sm.qs[h * HD + c * 8]);
                    const float4 qb = *reinterpret_cast<const float4*>(&sm.qs[h * HD + c * 8 + 4]);
                    float t = sa[h][i & 1], u = sb[h][i & 1];
                    t = fmaf(qa.x, bf_lo(wa.x), t); u = fmaf(qa.x, bf_lo(wb.x), u);
                    t = fmaf(qa.y, bf_hi(wa.x), t); u = fmaf(qa.y, bf_hi(wb.x), u);
                    t = fmaf(qa.z, bf_lo(wa.y), t); u = fmaf(qa.z, bf_lo(wb.y), u);
                    t = fmaf(qa.w, bf_hi(wa.y), t); u = fmaf(qa.w, bf_hi(wb.y), u);
                    t = fmaf(qb.x, bf_lo(wa.z), t); u = fmaf(qb.x, bf_lo(wb.z), u);
                    t = fmaf(qb.y, bf_hi(wa.z), t); u = fmaf(qb.y, bf_hi(wb.z), u);
                    t = fmaf(qb.z, bf_lo(wa.w), t); u = fmaf(qb.z, bf_lo(wb.w), u);
                    t = fmaf(qb.w, bf_hi(wa.w), t); u = fmaf(qb.w, bf_hi(wb.w), u);
                    sa[h][i & 1] = t;
                    sb[h][i & 1] = u;
                }
            }
        }
        float pa[GMAX], pb[GMAX];
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            pa[h] = pb[h] = 0.f;
            if (h < r) {
                float s0 = sa[h][0] + sa[h][1], s1 = sb[h][0] + sb[h][1];
                s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                if (!ma) s0 = -INFINITY;
                if (!mb) s1 = -INFINITY;
                float mx = fmaxf(s0, s1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mn = fmaxf(m[h], mx);  // finite: na >= 1
                const float corr = exp2f(m[h] - mn);
                const float e0 = exp2f(s0 - mn), e1 = exp2f(s1 - mn);
                float ps = e0 + e1;
                ps += __shfl_xor_sync(0xffffffffu, ps, 4);
                ps += __shfl_xor_sync(0xffffffffu, ps, 8);
                ps += __shfl_xor_sync(0xffffffffu, ps, 16);
                lsum[h] = fmaf(lsum[h], corr, ps);
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] *= corr;
                m[h] = mn;
                pa[h] = e0;
                pb[h] = e1;
            }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            float v0[E], v1[E];
            if (jj < na) ld_v<E>(va + (size_t)jj * HD + lane * E, v0);
            if (jj < nb) ld_v<E>(vb + (size_t)jj * HD + lane * E, v1);
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                if (h < r) {
                    const float p0 = __shfl_sync(0xffffffffu, pa[h], jj * 4);
                    const float p1 = __shfl_sync(0xffffffffu, pb[h], jj * 4);
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        if (jj < na) acc[h][e] = fmaf(p0, v0[e], acc[h][e]);
                        if (jj < nb) acc[h][e] = fmaf(p1, v1[e], acc[h][e]);
                    }
                }
            }
        }
    };

    // Within a stage, warp gw takes positions [n * gw / 8, n * (gw + 1) / 8): at most 8 with
    // hd 128, at most 16 (the two blocks of one pass) with hd 64. With hd 128 a warp takes two
    // stages per pass, one block from each, so each online-softmax update covers 16 positions.
    static_assert(kGroups == 1, "attention stages assume one consumer group");
    const int nst = at.nst;
    const int gw = warp % kGroupWarps;
    unsigned long long& waited = tr.waited;
    auto slice = [&](const Ring& at_rg, int j, const __nv_bfloat16*& k, const __nv_bfloat16*& v) {
        const int s0 = at.a + j * P.pos_per_stage;
        const int n = min(P.pos_per_stage, at.tma_end - s0);
        const __nv_bfloat16* st = reinterpret_cast<const __nv_bfloat16*>(sm.ring + (size_t)at_rg.slot * kStageBytes);
        const int p0 = n * gw / kGroupWarps, p1 = n * (gw + 1) / kGroupWarps;
        k = st + (size_t)p0 * HD;
        v = st + (size_t)(n + p0) * HD;
        return p1 - p0;
    };
    for (int j = 0; j < nst;) {
        const Ring ra = rg;
        rg.advance(P.ns);
        const bool two = HD == 128 && j + 1 < nst;
        const Ring rb = rg;
        if (two) rg.advance(P.ns);
        if (ok) {
            if (!wait_full(sm, ra, P, ctl, waited) || (two && !wait_full(sm, rb, P, ctl, waited))) {
                ok = false;
            } else {
                const __nv_bfloat16 *ka, *va, *kb, *vb;
                int na = slice(ra, j, ka, va), nb = 0;
                if (two) {
                    nb = slice(rb, j + 1, kb, vb);
                } else {  // hd 64: the stage's second block of 8
                    nb = na > 8 ? na - 8 : 0;
                    na -= nb;
                    kb = ka + (size_t)8 * HD, vb = va + (size_t)8 * HD;
                }
                if (na == 0 && nb > 0) {  // pass2 wants a non-empty first block
                    ka = kb, va = vb, na = nb, nb = 0;
                }
                if (na > 0) pass2(ka, va, na, kb, vb, nb);
                __syncwarp();
                if (lane == kSyncLane) {
                    mbar_arrive(smem_u32(&sm.empty[ra.slot]));
                    if (two) mbar_arrive(smem_u32(&sm.empty[rb.slot]));
                }
            }
        }
        j += two ? 2 : 1;
    }
    // merge the warps' states (and the current position's record)
    if (tid == 0) tr.mark(5);
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
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
    const int nrec = kConsumerWarps + (has_current ? 1 : 0);
    for (int idx = tid; idx < r * HD; idx += kConsumerThreads) {
        const int h = idx / HD, dd = idx % HD;
        float M = -INFINITY;
        for (int w = 0; w < nrec; ++w) M = fmaxf(M, ws[((size_t)w * r + h) * rec]);
        float L = 0.f, o = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < nrec; ++w) {
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
        // one acquire-release add: publishes this CTA's partial records (ordered before it by
        // the barrier above) and, for the last piece to arrive, makes everyone else's visible
        unsigned int* cnt = reinterpret_cast<unsigned int*>(ctl + kCtlHead + 16 * at.g);
        const unsigned int old = atom_add_acq_rel_u32(cnt, 1u);
        sm.flag[1] = ((old + 1u) % (unsigned)A) == 0u;
    }
    consumer_sync();
    if (sm.flag[1]) {  // last piece of this kv head to finish: combine all pieces
        // Each thread owns output (h, dd) and reads (m_i, l_i, acc_i[dd]) of the pieces in
        // batches of kCombineBatch, all loads of a batch in flight together, folding each
        // batch in with the usual max-rescaled sum (pieces in ascending order).
        const float* hp = part + (size_t)at.g * A * r * rec;
        unsigned long long* og = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.o) +
                                 (size_t)at.g * r * HD;
        const size_t stride = (size_t)r * rec;
        for (int idx = tid; idx < r * HD; idx += kConsumerThreads) {
            const int h = idx / HD, dd = idx % HD;
            const float* src = hp + (size_t)h * rec;
            float M = -INFINITY, L = 0.f, o = 0.f;
            for (int i0 = 0; i0 < A; i0 += kCombineBatch) {
                float mi[kCombineBatch], li[kCombineBatch], ai[kCombineBatch];
#pragma unroll
                for (int k = 0; k < kCombineBatch; ++k) {
                    mi[k] = -INFINITY, li[k] = 0.f, ai[k] = 0.f;  // pieces past A weigh nothing
                    if (i0 + k < A) {
                        const float* pr = src + (size_t)(i0 + k) * stride;
                        mi[k] = __ldcg(pr), li[k] = __ldcg(pr + 1), ai[k] = __ldcg(pr + 2 + dd);
                    }
                }
                float Mb = M;
#pragma unroll
                for (int k = 0; k < kCombineBatch; ++k) Mb = fmaxf(Mb, mi[k]);
                if (Mb != -INFINITY) {  // else no position in these pieces yet
                    const float c = exp2f(M - Mb);  // 0 when M is still -inf
                    L *= c, o *= c;
#pragma unroll
                    for (int k = 0; k < kCombineBatch; ++k) {
                        const float f = exp2f(mi[k] - Mb);  // 0 for an empty or absent piece
                        L = fmaf(li[k], f, L);
                        o = fmaf(ai[k], f, o);
                    }
                    M = Mb;
                }
            }
            st_tagged(og + (size_t)h * HD + dd, o / L, sc.tag);
        }
        if (tid == 0) tr.mark(7);
    }
    rg_ref = rg;
    ok_ref = ok;
}

// ------------------------------------------------------------------ producer

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Walks this CTA's stages in consumption order: steps, layers, phases, stages.
struct Cursor {
    int t = 0, l = 0, ph = 0, j = 0, nst = 0;
    bool done = false;
    const int* geom = nullptr;  // cta_geometry
    int at_t = -1;              // step whose attention piece `at` holds
    Gemv g;
    Attn at;

    __device__ void begin(const Params& P) {
        done = P.steps <= 0;
        if (!done) enter(P);
        settle(P);
    }
    __device__ void enter(const Params& P) {
        j = 0;
        if (ph == kATT) {
            if (at_t != t) {  // once per step: the piece only moves with the position
                at = attn_geom(P, P.pos0 + t, blockIdx.x);
                at_t = t;
            }
            nst = at.g < 0 ? 0 : at.nst;
        } else {
            g = gemv_geom(P, geom, ph, ph == kLM ? 0 : l);
            nst = g.nst;
        }
    }
    __device__ void settle(const Params& P) {
        while (!done && j >= nst) {
            if (ph < kD) {
                ++ph;
            } else if (ph == kD && l + 1 < P.dm.L) {
                ++l;
                ph = kQKV;
            } else if (ph == kD && step_has_head(P, t)) {
                ph = kLM;
            } else {
                ++t;
                l = 0;
                ph = kQKV;
                if (t >= P.steps) {
                    done = true;
                    return;
                }
            }
            enter(P);
        }
    }
    __device__ void next(const Params& P) {
        ++j;
        settle(P);
    }
    // Source ranges of the current stage; kv_last >= 0 is the last cache position it reads.
    __device__ void stage(const Params& P, const void*& s1, uint32_t& b1, const void*& s2, uint32_t& b2,
                          int& kv_last) const {
        if (ph == kATT) {
            const Dims& dm = P.dm;
            const int s0 = at.a + j * P.pos_per_stage;
            const int n = min(P.pos_per_stage, at.tma_end - s0);
            const size_t row = (((size_t)l * dm.Hkv + at.g) * dm.S + s0) * dm.hd;
            s1 = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.kcache) + row;
            s2 = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.vcache) + row;
            b1 = b2 = (uint32_t)((size_t)n * dm.hd * 2);
            kv_last = s0 + n - 1;
        } else {
            const size_t rowb = (size_t)g.K * 2;
            const int r0 = g.row0 + j * g.R;
            const int n = min(g.R, g.row1 - r0);
            s1 = g.base + (size_t)r0 * rowb;
            b1 = (uint32_t)(n * rowb);
            s2 = nullptr;
            b2 = 0;
            kv_last = -1;
        }
    }
};

struct Producer {
    const Params& P;
    const Smem sm;
    unsigned long long* ctl;
    uint64_t base;
    uint64_t policy;
    int k = 0;               // stages issued
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

    // Keep at most P.inflight issued stages in flight: wait until stage k - inflight has
    // landed. (Its slot cannot have been refilled yet, so its full-barrier phase is unambiguous.)
    __device__ bool wait_landed() {
        const int kk = k - P.inflight;
        if (P.inflight <= 0 || kk < 0 || P.inflight >= P.ns) return true;
        const uint32_t a = smem_u32(&sm.full[kk % P.ns]);
        const uint32_t par = (uint32_t)((kk / P.ns) & 1);
        if (mbar_try_wait(a, par)) return true;
        const uint64_t t0 = globaltimer();
        for (;;) {
            if (mbar_wait_hint(a, par)) return true;
            if (read_status(ctl) != 0) return false;
            if (globaltimer() - t0 > (uint64_t)P.timeout_ns) {
                raise_timeout(ctl, where_code(kWhereEmpty, 0x80 | (kk % P.ns)));
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

    __device__ bool issue(const Cursor& cur) {
        const void *s1, *s2;
        uint32_t b1, b2;
        int kv_last;
        cur.stage(P, s1, b1, s2, b2, kv_last);
        if (kv_last >= P.pos0) {  // written earlier in this launch: wait for the grid barrier
            // that ends the step that appended it (the attention phase writes the row)
            if (!wait_epochs((long long)(kv_last - P.pos0) + 1)) return false;
        }
        if (!wait_landed()) return false;
        if (!wait_empty()) return false;
        const uint32_t fb = smem_u32(&sm.full[slot]);
        const uint32_t dst = smem_u32(sm.ring + (size_t)slot * kStageBytes);
        mbar_expect_tx(fb, b1 + b2);
        bulk_g2s(dst, s1, b1, fb, policy);
        if (b2) bulk_g2s(dst + b1, s2, b2, fb, policy);
        ++k;
        if (++slot == P.ns) {
            slot = 0;
            ++pass;
        }
        return true;
    }

    // Pull a later stage's bytes into L2 ahead of time; no shared memory, no completion to
    // track, and harmless if a line is written afterwards (L2 is the coherence point).
    __device__ void prefetch(const Cursor& cur) {
        const void *s1, *s2;
        uint32_t b1, b2;
        int kv_last;
        cur.stage(P, s1, b1, s2, b2, kv_last);
        bulk_prefetch_l2(s1, b1);
        if (b2) bulk_prefetch_l2(s2, b2);
    }

    __device__ void run() {
        const long long c_start = clock64();
        bool ok = true;
        Cursor ld, pf;
        ld.geom = pf.geom = sm.geom;
        ld.begin(P);
        pf.begin(P);
        // The L2 lookahead (off unless requested) runs a second cursor P.prefetch stages ahead.
        const bool lookahead = P.prefetch > 0;
        for (int i = 0; i < P.prefetch && !pf.done; ++i, pf.next(P)) prefetch(pf);
        while (ok && !ld.done) {
            if (lookahead && !pf.done) {
                prefetch(pf);
                pf.next(P);
            }
            ok = issue(ld);
            ld.next(P);
        }
        // Let every copy already issued land before the CTA exits: when the consumers have
        // stopped early (a refused token, a wait that gave up) nobody else waits for them.
        // On a normal run these stages were consumed already and each test passes at once.
        // The bound is fixed and generous, not the launch's wait limit (which may be tiny):
        // an issued copy always completes within microseconds.
        {
            constexpr uint64_t kDrainNs = 100000000ull;  // 100 ms
            const int first = k > P.ns ? k - P.ns : 0;
            for (int kk = first; kk < k; ++kk) {
                const uint32_t a = smem_u32(&sm.full[kk % P.ns]);
                const uint32_t par = (uint32_t)((kk / P.ns) & 1);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(a, par) && globaltimer() - t0 < kDrainNs) {
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

// One instantiation per attention shape (head dim, q heads per kv head rounded up to 2, 4
// or 8), so the fully inlined kernel holds one attention body and its registers.
template <int HD, int GMAX, int MAXCH>
__global__ void __launch_bounds__(kThreads, 1) monokernel(const __grid_constant__ Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem sm = carve(P, smem_raw);
    unsigned long long* ctl = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.ctl);
    const int tid = threadIdx.x;
    const Dims& dm = P.dm;

    if (tid == 0) {
        for (int s = 0; s < P.ns; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), kGroupWarps);  // every warp of the slot's group releases
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        cta_geometry(P, blockIdx.x, sm.geom);
        // Barrier count at launch: a multiple of nb plus arrivals of CTAs that already
        // reached this launch's first barrier (which cannot complete before we arrive).
        const uint64_t raw = ld_acquire_u64(ctl + kCtlBar);
        reinterpret_cast<unsigned long long*>(sm.flag)[kFlagBase] = raw - raw % (uint64_t)P.nb;
        reinterpret_cast<unsigned long long*>(sm.flag)[kFlagEpoch] = 0ull;
        sm.flag[0] = read_status(ctl);
        if (blockIdx.x == 0) ctl[kCtlArgmax] = 0ull;  // step 0's argmax slot
    }
    __syncthreads();
    const uint64_t base = reinterpret_cast<unsigned long long*>(sm.flag)[kFlagBase];
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
    const unsigned long long* tagged = reinterpret_cast<const unsigned long long*>(P.arena);
    const __nv_bfloat16* embed = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.embed);
    Ring rg;
    StepCtx sc;
    bool ok = true;
    Tracer tr;
    if (P.trace && tid == 0 && blockIdx.x % P.trace_every == 0) {
        tr.row0 = P.trace + (size_t)(blockIdx.x / P.trace_every) * P.trace_rows * kTraceWords;
        tr.rows = P.trace_rows;
        tr.mark(0);
    }

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
            // A token id outside the vocabulary (a bad pending input) stops the launch before
            // the embedding row is read. Every CTA reads the same id, so all of them stop here.
            if ((unsigned)tok >= (unsigned)dm.V) {
                raise_status(ctl, kStatusToken, where_code(kWhereToken, t));
                tok = -1;
            }
            sm.flag[2] = tok;
        }
        if (tid == 32) *sm.att = attn_geom(P, sc.p, blockIdx.x);  // this step's attention piece
        if (tid < dm.hd / 2)  // this position's RoPE row (cos, sin per pair)
            sm.rope[tid] = __ldg(reinterpret_cast<const float2*>(P.arena + P.lay.rope) + (size_t)sc.p * (dm.hd / 2) + tid);
        consumer_sync();
        const int tok = sm.flag[2];
        if (tok < 0) {
            ok = false;
            break;
        }
        {
            const __nv_bfloat16* erow = embed + (size_t)tok * dm.d;
            const int own0 = sm.geom[kGeomOwn], own1 = sm.geom[kGeomOwn + 1];
            for (int i = own0 + tid; i < own1; i += kConsumerThreads)
                sm.xown[i - own0] = __bfloat162float(erow[i]);  // the residual rows this CTA updates in O and D
        }

        // The step's phases in order: per layer QKV, ATT, O, GU, D, then the LM head if this
        // step's logits are needed. One loop with one call site per phase kind keeps the
        // (fully inlined) kernel's code and register allocation to one copy of each. Every
        // phase's input is the previous phase's tagged output (the first QKV reads the
        // embedding row), so phases follow each other without grid barriers; one barrier
        // ends the step (the argmax and the KV rows appended this step are then complete).
        const int nphase = 5 * dm.L + (step_has_head(P, t) ? 1 : 0);
        for (int q = 0; q < nphase; ++q) {
            const int l = q / 5 < dm.L ? q / 5 : 0;
            const int ph = q / 5 < dm.L ? q % 5 : kLM;
            sc.l = l;
            sc.tag = phase_tag(P, t, q);
            const uint32_t tag_in = sc.tag - 1u;  // the previous phase's
            const uint8_t* lb = P.arena + P.lay.layer0 + (size_t)l * P.lay.layer_stride;
            // this phase's input vector -> xs
            if (ph == kO) {
                load_vector(sm, tagged + P.lay.o / 8, tag_in, dm.qd, P, ctl, ok);
            } else if (ph == kD) {
                load_vector(sm, tagged + P.lay.gu / 8, tag_in, dm.F, P, ctl, ok);
            } else if (ph != kATT) {
                const __nv_bfloat16* gain = reinterpret_cast<const __nv_bfloat16*>(
                    ph == kQKV ? lb + P.lay.l_attn_norm : ph == kGU ? lb + P.lay.l_ffn_norm : P.arena + P.lay.final_norm);
                const bool from_embed = ph == kQKV && l == 0;
                const unsigned long long* xin = tagged + P.lay.x / 8 + (ph == kGU ? 0 : dm.d);  // O's or D's output
                const __nv_bfloat16* erow = embed + (size_t)sm.flag[2] * dm.d;  // this step's token row
                load_rmsnorm(sm, from_embed ? nullptr : xin, tag_in, from_embed ? erow : nullptr, gain, dm.d, dm.eps, P,
                             ctl, ok);
            }
            if (tid == 0) tr.mark(1);
            if (ph == kATT) {
                run_attention<HD, GMAX>(P, sm, ctl, l, rg, sc, ok, tr);
            } else {
                run_gemv<MAXCH>(P, sm, ctl, ph, l, rg, sc, ok, tr);
            }
            if (ph == kLM) {
                if ((tid & 31) == 0) sm.best[tid >> 5] = sc.lm_best;
                consumer_sync();
                if (tid == 0 && ok) {
                    unsigned long long b = 0ull;
                    for (int w = 0; w < kConsumerWarps; ++w) b = sm.best[w] > b ? sm.best[w] : b;
                    atomicMax(ctl + kCtlArgmax + 16 * (t % 3), b);
                }
            }
            if (q + 1 < nphase) {
                if (!(ok = phase_end(ok, tr))) break;
            } else {
                if (!(ok = grid_sync(sm, P, ctl, ok, tr))) break;
            }
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

template <int MAXCH>
static const void* kernel_for_ch(int hd, int r) {
    if (hd == 128) {
        if (r <= 2) return (const void*)monokernel<128, 2, MAXCH>;
        if (r <= 4) return (const void*)monokernel<128, 4, MAXCH>;
        return (const void*)monokernel<128, 8, MAXCH>;
    }
    if (r <= 2) return (const void*)monokernel<64, 2, MAXCH>;
    if (r <= 4) return (const void*)monokernel<64, 4, MAXCH>;
    return (const void*)monokernel<64, 8, MAXCH>;
}
static const void* kernel_for(const Dims& dm) {
    return gemv_max_chunks(dm) <= 4 ? kernel_for_ch<4>(dm.hd, dm.r) : kernel_for_ch<8>(dm.hd, dm.r);
}

int monokernel_occupancy(const Dims& dm, int smem_bytes, int* blocks_per_sm) {
    const void* k = kernel_for(dm);
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return (int)e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, k, kThreads, smem_bytes);
    return (int)e;
}

void launch_decode(const Params& p, void* stream, int smem_bytes, int* err) {
    void* args[] = {const_cast<Params*>(&p)};
    cudaError_t e = cudaLaunchCooperativeKernel(kernel_for(p.dm), dim3(p.nb), dim3(kThreads), args,
                                                (size_t)smem_bytes, (cudaStream_t)stream);
    *err = (int)e;
}

}  // namespace kd
