// kd_kernel.cu -- the decode monokernel: one persistent cooperative launch per kd_decode
// that runs every decode step of the request, layer after layer, without returning to the
// host ("3000 tokens per second: how to speed up LLMs on ordinary GPUs", aikraft.ru,
// section 04 "Monokernel and optimized GPU code": one resident GPU program covering matrix
// products, attention, normalisation and sampling, with tight control of synchronisation,
// prefetch and execution order).
//
// B200 design (one CTA per SM, 148 CTAs, 1 producer warp + 16 consumer warps each):
//  * Weight streaming. The producer warp walks the CTA's fixed schedule of weight rows and
//    KV-cache rows and streams them HBM -> shared memory with 1-D bulk async copies
//    (cp.async.bulk) into a ring of 32 KB stages guarded by mbarriers. Weights never depend
//    on activations, so the ring fills while the consumers wait for their inputs: waits
//    are absorbed instead of leaving HBM idle (the pages name prefetch and synchronisation
//    control as the monokernel's levers, aikraft.ru section 04; the per-token time budget
//    that makes each microsecond count is their section 03).
//  * Batch-1 decode is a matrix-vector product (about 1 FLOP per weight byte, their
//    section 02), so there are no tensor-core tiles: 16-byte bf16 loads from shared
//    memory, fp32 FMAs, warp-shuffle reductions.
//  * Two cross-CTA sums per layer. The output projection and the down projection are
//    split over their reduction dimension (split-K): each CTA multiplies the attention
//    output dims or the hidden units it produced itself by the matching transposed weight
//    rows and adds its partial d-vector into one of two zeroed copies of the sum with vector
//    atomics, then arrives on a monotonic 64-bit counter (one copy of it on each of the
//    B200's two dies). Every CTA keeps the whole residual stream in shared memory and folds
//    the sum in once the counter reaches its target.
//  * Group-local exchanges. The CTAs of one kv head compute that head's Q/K/V rows, its
//    attention pieces and its output-projection columns, so the Q/K/V -> attention and
//    attention -> output-projection hand-offs only wait for sibling CTAs. They pass 64-bit
//    tagged words (fp32 value + phase tag in one single-copy-atomic store): a reader polls
//    the data itself, no barrier or flag.
//  * Attention is split-K over the cached positions (pieces of one kv head per CTA). A
//    piece scores a block of positions, takes the block's softmax statistics once, then
//    accumulates V, and publishes (max, sum, acc) records; the output-projection CTAs of the
//    head combine the records of every piece for their own columns.
//  * The LM head ends in a packed (value, index) atomicMax; every CTA reads the winner
//    and gathers the next embedding row itself, so sampling never leaves the GPU
//    (agentlenshq.com "Breaking the memory wall", section "1. The Monokernel Runtime").
//  * Every wait is bounded by a time limit and unwinds with an error status instead of
//    hanging.
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
// Parity wait with a hardware suspend hint: the warp sleeps until the phase completes or
// the hint expires instead of spinning.
__device__ __forceinline__ bool mbar_wait_hint(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(a), "r"(parity), "r"(20000u)
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
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}
__device__ __forceinline__ void red_max_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ float4 ld_relaxed_v4(const float* p) {
    float4 v;
    asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Tagged activation words: value (fp32 bits) in the low half, the producing phase's tag in
// the high half. A 64-bit store is single-copy atomic, so a reader that sees the tag sees
// the value written with it; no fence or barrier orders the two.
__device__ __forceinline__ unsigned long long tag_word(float v, uint32_t tag) {
    return ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
}
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, uint32_t tag) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(tag_word(v, tag)) : "memory");
}
__device__ __forceinline__ unsigned long long ld_tagged(const unsigned long long* p) {
    unsigned long long w;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}
__device__ __forceinline__ float tagged_value(unsigned long long w) { return __uint_as_float((uint32_t)w); }
__device__ __forceinline__ bool tagged_is(unsigned long long w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }

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
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ int read_status(const unsigned long long* ctl) {
    return static_cast<int>(*reinterpret_cast<const volatile unsigned long long*>(ctl + kCtlStatus));
}
// The first error of a launch wins: its code goes to the status word, its place to kCtlWhere.
__device__ __noinline__ void raise_status(unsigned long long* ctl, int code, int where) {
    if (atomicCAS(ctl + kCtlStatus, 0ull, (unsigned long long)code) == 0ull)
        atomicExch(ctl + kCtlWhere, (unsigned long long)where);
}

// Where a wait gave up or an input was refused: (what << 24) | (cta << 8) | detail.
enum { kWhereFull = 1, kWhereEmpty = 2, kWhereSync = 3, kWhereKv = 4, kWhereToken = 5, kWhereData = 6 };
__device__ __forceinline__ int where_code(int what, int detail) {
    return (what << 24) | ((int)blockIdx.x << 8) | (detail & 0xff);
}

// Time limit shared by every bounded wait of one thread: started at the first miss.
struct Deadline {
    uint64_t t0 = 0;
    // true while the wait may continue; false (status raised) once the limit has passed or
    // another wait of the launch has failed
    __device__ __forceinline__ bool alive(const unsigned long long* ctl, long long limit, int where) {
        if (read_status(ctl) != 0) return false;
        const uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        if (now - t0 > (uint64_t)limit) {
            raise_status(const_cast<unsigned long long*>(ctl), kStatusTimeout, where);
            return false;
        }
        return true;
    }
};

// Per-phase timestamps (SM cycles) of one CTA, recorded by consumer thread 0.
struct Tracer {
    unsigned long long* row0 = nullptr;
    int row = 0, rows = 0;
    unsigned long long waited = 0;  // cycles spent waiting for stages in this phase
    __device__ __forceinline__ void mark(int col) {
        if (row0 && row < rows - 1) row0[(size_t)row * kTraceWords + col] = (unsigned long long)clock64();
    }
    __device__ __forceinline__ void begin(int id) {
        if (row0 && row < rows - 1) {
            row0[(size_t)row * kTraceWords] = (unsigned long long)id;
            row0[(size_t)row * kTraceWords + 6] = 0ull;
            row0[(size_t)row * kTraceWords + 7] = 0ull;
            mark(1);
        }
    }
    // stage j of nst of the phase has landed: the first and the last one are stamped
    __device__ __forceinline__ void stage_ready(int j, int nst) {
        if (j == 0) mark(6);
        if (j == nst - 1) mark(7);
    }
    __device__ __forceinline__ void end() {
        if (row0 && row < rows - 1) {
            mark(4);
            row0[(size_t)row * kTraceWords + 5] = waited;
        }
        waited = 0;
        ++row;
    }
};

// ------------------------------------------------------------------ schedule geometry
// The producer and the consumers enumerate the same stage sequence from these.

enum Phase { kQKV = 0, kATT = 1, kO = 2, kGU = 3, kD = 4, kLM = 5 };

// This CTA's share of every phase, computed once per launch into shared memory.
struct Geo {
    int grp, piece;  // kv head and piece index (grp < 0: no Q/K/V rows, attention piece or O columns)
    int q0, q1;      // rows of the kv-head-major Q/K/V matrix
    int o0, o1;      // attention output dims (rows of the transposed output projection)
    int u0, u1;      // hidden units (gate/up row pairs, rows of the transposed down projection)
    int v0, v1;      // LM-head rows
};
__device__ void cta_geo(const Params& P, int c, Geo& g) {
    const Dims& dm = P.dm;
    const int A = P.pieces;
    if (c < A * dm.Hkv) {
        g.grp = c / A;
        g.piece = c % A;
        const int pairs = (dm.r + 2) * dm.hd / 2;  // RoPE pairs (and v pairs) of one kv head's rows
        const int base = g.grp * (dm.r + 2) * dm.hd;
        g.q0 = base + 2 * (pairs * g.piece / A);
        g.q1 = base + 2 * (pairs * (g.piece + 1) / A);
        const int cc = dm.r * dm.hd;  // attention output dims of the kv head's q heads
        g.o0 = g.grp * cc + cc * g.piece / A;
        g.o1 = g.grp * cc + cc * (g.piece + 1) / A;
    } else {
        g.grp = -1;
        g.piece = 0;
        g.q0 = g.q1 = g.o0 = g.o1 = 0;
    }
    g.u0 = (int)((long long)dm.F * c / P.nb);
    g.u1 = (int)((long long)dm.F * (c + 1) / P.nb);
    g.v0 = (int)((long long)dm.V * c / P.nb);
    g.v1 = (int)((long long)dm.V * (c + 1) / P.nb);
}

// This CTA's attention piece at position p: the T = p + 1 positions of its kv head are cut
// into `pieces` contiguous ranges; the last one also holds p, whose K and V come from this
// step's Q/K/V words instead of the cache.
struct Piece {
    int a, e;  // cached positions [a, e), streamed through the ring
    int cur;   // 1 if position p belongs to this piece
    int nblk;  // softmax blocks of at most `blk` cached positions (at least 1 when cur)
};
__device__ __forceinline__ Piece piece_geo(const Params& P, int piece, int p) {
    Piece pc;
    const long long T = (long long)p + 1;
    const int A = P.pieces;
    pc.a = (int)(T * piece / A);
    const int b = (int)(T * (piece + 1) / A);
    pc.cur = b == (int)T;
    pc.e = pc.cur ? p : b;
    pc.nblk = (pc.e - pc.a + P.blk - 1) / P.blk;
    if (pc.cur && pc.nblk == 0) pc.nblk = 1;
    return pc;
}
// Cached positions of block kb of a piece.
__device__ __forceinline__ int block_len(const Params& P, const Piece& pc, int kb) {
    const int s = pc.a + kb * P.blk;
    const int n = pc.e - s;
    return n < 0 ? 0 : (n > P.blk ? P.blk : n);
}

// The LM head runs at steps that pick a token, or at every step when logits are dumped.
__device__ __forceinline__ bool step_has_head(const Params& P, int t) {
    return P.dump || t >= P.n_pending - 1;
}
// Tags of the Q/K/V words and the attention records of step t, layer l.
__device__ __forceinline__ uint32_t qkv_tag(const Params& P, int t, int l) {
    return P.tag0 + 1u + 2u * (uint32_t)(t * P.dm.L + l);
}

// ------------------------------------------------------------------ shared memory

struct Smem {
    uint8_t* ring;            // ns * kStageBytes
    float* x;                 // the residual stream (d), identical in every CTA
    __nv_bfloat16* gain;      // the norm gain of the next row GEMV (d), prefetched
    float* hin;               // split-K inputs: this CTA's hidden values or attention output dims
    float* work;              // GEMV row partials / attention scores and reductions / split-K sums
    float* qs;                // attention: q of the kv head's q heads (r * hd), prescaled
    float* kvc;               // attention: the current position's k and v (2 * hd), bf16 values
    float2* rope;             // (cos, sin) for hd/2 frequencies at this step's position
    float* red;               // reduction scratch (kConsumerWarps * 8)
    float* stats;             // attention running max and sum per q head (2 * kMaxGroup)
    unsigned long long* u64;  // [0] sync count at launch, [1] the local counter copy, [2] the other copy
    int* flag;                // broadcast slots
    uint64_t* full;           // mbarriers
    uint64_t* empty;
    Geo* geo;
    Piece* piece;             // this step's attention piece (written at the step start)
};

// Byte offsets of the shared-memory regions; the ring starts at 0 (1024-aligned), the others
// on 128-byte boundaries. Used by the kernel and for the launch size.
struct SmemLayout {
    size_t ring, x, gain, hin, work, qs, kvc, rope, red, stats, u64, flag, full, empty, geo, piece, total;
};
__host__ __device__ inline SmemLayout smem_layout(int ns, int d, int hd, int r, int hin_floats, int work_floats) {
    SmemLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = (off + bytes + 127) & ~(size_t)127;
        return at;
    };
    L.ring = take((size_t)ns * kStageBytes);
    L.x = take((size_t)d * 4);
    L.gain = take((size_t)d * 2);
    L.hin = take((size_t)hin_floats * 4);
    L.work = take((size_t)work_floats * 4);
    L.qs = take((size_t)r * hd * 4);
    L.kvc = take((size_t)2 * hd * 4);
    L.rope = take((size_t)hd / 2 * 8);
    L.red = take((size_t)kConsumerWarps * 8 * 4);
    L.stats = take((size_t)2 * kMaxGroup * 4);
    L.u64 = take(4 * 8);
    L.flag = take(16 * 4);
    L.full = take((size_t)kMaxStages * 8);
    L.empty = take((size_t)kMaxStages * 8);
    L.geo = take(sizeof(Geo));
    L.piece = take(sizeof(Piece));
    L.total = off;
    return L;
}

__device__ __forceinline__ Smem carve(const Params& P, uint8_t* base) {
    const SmemLayout L = smem_layout(P.ns, P.dm.d, P.dm.hd, P.dm.r, P.hin_floats, P.work_floats);
    Smem s;
    s.ring = base + L.ring;
    s.x = reinterpret_cast<float*>(base + L.x);
    s.gain = reinterpret_cast<__nv_bfloat16*>(base + L.gain);
    s.hin = reinterpret_cast<float*>(base + L.hin);
    s.work = reinterpret_cast<float*>(base + L.work);
    s.qs = reinterpret_cast<float*>(base + L.qs);
    s.kvc = reinterpret_cast<float*>(base + L.kvc);
    s.rope = reinterpret_cast<float2*>(base + L.rope);
    s.red = reinterpret_cast<float*>(base + L.red);
    s.stats = reinterpret_cast<float*>(base + L.stats);
    s.u64 = reinterpret_cast<unsigned long long*>(base + L.u64);
    s.flag = reinterpret_cast<int*>(base + L.flag);
    s.full = reinterpret_cast<uint64_t*>(base + L.full);
    s.empty = reinterpret_cast<uint64_t*>(base + L.empty);
    s.geo = reinterpret_cast<Geo*>(base + L.geo);
    s.piece = reinterpret_cast<Piece*>(base + L.piece);
    return s;
}

int monokernel_smem_bytes(const Params& p) {
    return (int)smem_layout(p.ns, p.dm.d, p.dm.hd, p.dm.r, p.hin_floats, p.work_floats).total;
}

// ------------------------------------------------------------------ ring and waits

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

// Wait (whole warp) for the stage in `rg` to land. Only lane 0 polls the mbarrier (sixteen
// warps times 32 lanes polling one shared-memory word would serialise on it); the shuffle
// hands its answer to the warp and the warp barrier orders the other lanes' reads of the
// stage after lane 0's observation of the completed phase. `waited` accumulates the cycles
// spent (trace).
__device__ __forceinline__ bool wait_full(const Smem& sm, const Ring& rg, const Params& P, const unsigned long long* ctl,
                                          unsigned long long& waited) {
    const uint32_t a = smem_u32(&sm.full[rg.slot]);
    int done = 0;
    if ((threadIdx.x & 31) == 0) {
        done = mbar_try_wait(a, rg.phase);
        if (!done) {
            const long long c0 = clock64();
            Deadline dl;
            for (;;) {
                if (mbar_wait_hint(a, rg.phase)) {
                    done = 1;
                    waited += (unsigned long long)(clock64() - c0);
                    break;
                }
                if (!dl.alive(ctl, P.timeout_ns, where_code(kWhereFull, rg.slot))) break;
            }
        }
    }
    done = __shfl_sync(0xffffffffu, done, 0);
    __syncwarp();
    return done != 0;
}
// The warp is done with the stage: one arrival per warp on the slot's empty barrier.
__device__ __forceinline__ void release(const Smem& sm, const Ring& rg) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&sm.empty[rg.slot]));
}

// Poll one tagged word until it carries `tag` (the first read was issued by the caller
// together with its other loads). Returns false, with the device status set, after the
// time limit or when another wait of the launch has failed.
__device__ __noinline__ bool poll_word(const unsigned long long* p, uint32_t tag, unsigned long long& w, const Params& P,
                                       const unsigned long long* ctl, int what) {
    Deadline dl;
    for (uint32_t it = 1;; ++it) {
        w = ld_tagged(p);
        if (tagged_is(w, tag)) return true;
        if ((it & 31) == 0 && !dl.alive(ctl, P.timeout_ns, where_code(kWhereData, what))) return false;
    }
}
__device__ __forceinline__ bool get_word(const unsigned long long* p, uint32_t tag, unsigned long long& w, const Params& P,
                                         const unsigned long long* ctl, int what) {
    return tagged_is(w, tag) || poll_word(p, tag, w, P, ctl, what);
}

// Arrive at the next cross-CTA sync: every consumer thread's atomics of this phase are done
// (the CTA barrier), then thread 0 publishes them with the arrival: one release fence and an
// add of 1 on every copy of the counter.
__device__ __forceinline__ void sync_arrive(const Smem& sm) {
    consumer_sync();
    if (threadIdx.x == 0) {
        unsigned long long* local = reinterpret_cast<unsigned long long*>(sm.u64[1]);
        unsigned long long* other = reinterpret_cast<unsigned long long*>(sm.u64[2]);
        if (other) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            asm volatile("red.relaxed.gpu.global.add.u64 [%0], 1;" ::"l"(local) : "memory");
            asm volatile("red.relaxed.gpu.global.add.u64 [%0], 1;" ::"l"(other) : "memory");
        } else {
            red_release_add_u64(local, 1ull);
        }
    }
}
// Wait until every CTA has arrived at this launch's sync number k (thread 0 polls with
// acquire loads, the CTA barrier then orders every consumer thread after it). Returns
// false in every consumer thread when the wait gave up or another wait failed.
__device__ __noinline__ int sync_spin(const unsigned long long* ctl, const unsigned long long* counter, uint64_t target,
                                     long long timeout_ns, long long k) {
    Deadline dl;
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire_u64(counter) >= target) return 1;
        if ((it & 31) == 31 && !dl.alive(ctl, timeout_ns, where_code(kWhereSync, (int)(k & 0xff)))) return 0;
    }
}
__device__ __forceinline__ bool sync_wait(const Smem& sm, const Params& P, const unsigned long long* ctl, long long k,
                                          bool ok) {
    if (threadIdx.x == 0) {
        const uint64_t target = sm.u64[0] + (uint64_t)(k + 1) * (uint64_t)P.nb;
        sm.flag[0] = ok ? sync_spin(ctl, reinterpret_cast<const unsigned long long*>(sm.u64[1]), target, P.timeout_ns, k) : 0;
    }
    consumer_sync();
    return sm.flag[0] != 0;
}

// After sync k has completed: zero this CTA's slice of delta buffer (k - 1) % 3. Every CTA
// finished reading that buffer before it arrived at sync k, and the buffer takes atomics
// again (as the buffer of sync k + 2) only after sync k + 1 has completed, which orders these
// stores before them.
__device__ __forceinline__ void zero_previous(const Params& P, long long k) {
    if (k < 1) return;
    const int d = P.dm.d;
    const int n = kSumCopies * d;  // every copy of the buffer
    float* old = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.delta) + (size_t)((k - 1) % 3) * n;
    const int z0 = (int)((long long)n * blockIdx.x / P.nb), z1 = (int)((long long)n * (blockIdx.x + 1) / P.nb);
    for (int i = z0 + (int)threadIdx.x; i < z1; i += kConsumerThreads) old[i] = 0.f;
}
// Start copying the norm gain of the coming row GEMV into shared memory (asynchronously:
// it lands while the phase waits for its inputs). fold_norm waits for it.
__device__ __forceinline__ void prefetch_gain(const Smem& sm, const __nv_bfloat16* gain, int d) {
    for (int i = threadIdx.x; i < d / 8; i += kConsumerThreads) cp_async16(sm.gain + i * 8, gain + i * 8);
    cp_async_commit();
}

// The residual stream's update and its RMSNorm scale. With k >= 0 (sync k has completed),
// delta buffer k % 3 -- the sum of every CTA's split-K partials, its copies added in copy
// order -- is folded into the residual first, and this CTA's slice of the previous buffer is
// recycled. Returns
// 1 / sqrt(mean(x^2) + eps) of the result: every CTA sums the same values in the same
// order, so all of them get the same scale. Also completes the gain prefetch.
__device__ __forceinline__ float fold_norm(const Smem& sm, const Params& P, long long k) {
    const int d = P.dm.d;
    const float* src = reinterpret_cast<const float*>(P.arena + P.lay.delta) + (size_t)(k >= 0 ? k % 3 : 0) * kSumCopies * d;
    float ss = 0.f;
    for (int i = threadIdx.x * 4; i < d; i += kConsumerThreads * 4) {
        float4* xp = reinterpret_cast<float4*>(sm.x + i);
        float4 x = *xp;
        if (k >= 0) {
            float4 v = ld_relaxed_v4(src + i);
#pragma unroll
            for (int c = 1; c < kSumCopies; ++c) {  // the copies, added in copy order
                const float4 u = ld_relaxed_v4(src + (size_t)c * d + i);
                v.x += u.x, v.y += u.y, v.z += u.z, v.w += u.w;
            }
            x.x += v.x, x.y += v.y, x.z += v.z, x.w += v.w;
            *xp = x;
        }
        ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
    }
    if (k >= 0) zero_previous(P, k);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) sm.red[threadIdx.x >> 5] = ss;
    cp_async_wait_all();
    consumer_sync();
    const float4* r4 = reinterpret_cast<const float4*>(sm.red);
    const float4 a = r4[0], b = r4[1], c = r4[2], e = r4[3];  // the 16 warp sums, read at once
    const float tot = ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w)) + ((c.x + c.y) + (c.z + c.w)) +
                      ((e.x + e.y) + (e.z + e.w));
    return 1.0f / sqrtf(tot / (float)d + P.dm.eps);
}

// ------------------------------------------------------------------ row GEMV

// rows [row0, row0 + nrows) of a bf16 matrix with rows of d elements, times the normalised
// residual xn = x * scale * gain. A stage holds gr rows; each row is cut into gs slices and
// warp w takes slice w % gs of gm rows of every stage, with its activation slice in
// registers (NCH chunks of 8 per lane). Lane partials of four units are reduced together
// (two exchange levels that halve the values a lane holds, then three plain levels), and the
// unit sums go to work[row * gs + slice]; the caller sums the slices after a CTA barrier.
template <int NCH, int GM>
__device__ __forceinline__ void gemv_rows(const Params& P, const Smem& sm, const unsigned long long* ctl, int nrows,
                                          float scale, Ring& rg, bool& ok, Tracer& tr) {
    const int d = P.dm.d;
    const int gs = P.sh.gs, gr = P.sh.gr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lgs = __ffs(gs) - 1;  // gs is a power of 2
    const int sl = warp & (gs - 1);
    const int rw = warp >> lgs, rstep = kConsumerWarps >> lgs;
    const int slen = d >> lgs;
    const size_t rowbytes = (size_t)d * 2;
    const int nst = (nrows + gr - 1) / gr;

    // Lanes 4..7 of each quarter-warp read the second half of their 8 activations first, so
    // that each 16-byte load of a quarter-warp touches 8 different bank groups.
    float xr[NCH][8];
    const int hsw = (lane >> 2) & 1;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int k = sl * slen + (lane + 32 * i) * 8;
        const float4 f = *reinterpret_cast<const float4*>(sm.x + k + 4 * hsw);
        const float4 z = *reinterpret_cast<const float4*>(sm.x + k + 4 - 4 * hsw);
        const float4 a = hsw ? z : f, b = hsw ? f : z;
        const uint4 g = lds128(sm.gain + k);
        xr[i][0] = (a.x * scale) * bf_lo(g.x), xr[i][1] = (a.y * scale) * bf_hi(g.x);
        xr[i][2] = (a.z * scale) * bf_lo(g.y), xr[i][3] = (a.w * scale) * bf_hi(g.y);
        xr[i][4] = (b.x * scale) * bf_lo(g.z), xr[i][5] = (b.y * scale) * bf_hi(g.z);
        xr[i][6] = (b.z * scale) * bf_lo(g.w), xr[i][7] = (b.w * scale) * bf_hi(g.w);
    }
    const int loff = sl * slen * 2 + lane * 16;  // this lane's first chunk in a row; then +512 B each

    // Stages are taken in batches of SB = SG / 2 (two stages when GM == 1): the batch's
    // stages are awaited together and their dot products formed together, so the fixed
    // latency of a stage hand-off (mbarrier wait, loads, FMA chain, release) is paid once per
    // batch and the batch's units give each warp independent chains to interleave.
    // The lane partials of four units (SG = 4 / GM stages) are then reduced together: value i
    // belongs to stage j0 + i / GM and row rw + (i % GM) * rstep. After the last stage of the
    // phase the group may be short; its missing values are zero and are not written.
    constexpr int SG = 4 / GM;
    constexpr int SB = SG >= 2 ? 2 : 1;
    for (int j0 = 0; j0 < nst; j0 += SG) {
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = 0.f;
#pragma unroll
        for (int b0 = 0; b0 < SG; b0 += SB) {
            Ring rgs[SB];
            bool have[SB];
            bool all = true;
#pragma unroll
            for (int q = 0; q < SB; ++q) {
                const int j = j0 + b0 + q;
                have[q] = j < nst;
                rgs[q] = rg;
                if (have[q]) {
                    rg.advance(P.ns);
                    if (ok && wait_full(sm, rgs[q], P, ctl, tr.waited)) tr.stage_ready(j, nst);
                    else all = false;
                }
            }
            if (!all) ok = false;
#pragma unroll
            for (int q = 0; q < SB; ++q) {
                const int j = j0 + b0 + q;
                if (have[q] && ok) {
                    const uint8_t* st = sm.ring + (size_t)rgs[q].slot * kStageBytes;
                    const int nr = min(gr, nrows - j * gr);
#pragma unroll
                    for (int u = 0; u < GM; ++u) {
                        const int row = rw + u * rstep;
                        if (row < nr) {
                            const uint8_t* wl = st + row * rowbytes + loff;
                            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                            for (int i = 0; i < NCH; ++i) {
                                const uint4 w = lds128(wl + i * 512);
                                a0 = fmaf(bf_lo(w.x), xr[i][0], a0);
                                a1 = fmaf(bf_hi(w.x), xr[i][1], a1);
                                a2 = fmaf(bf_lo(w.y), xr[i][2], a2);
                                a3 = fmaf(bf_hi(w.y), xr[i][3], a3);
                                a0 = fmaf(bf_lo(w.z), xr[i][4], a0);
                                a1 = fmaf(bf_hi(w.z), xr[i][5], a1);
                                a2 = fmaf(bf_lo(w.w), xr[i][6], a2);
                                a3 = fmaf(bf_hi(w.w), xr[i][7], a3);
                            }
                            v[(b0 + q) * GM + u] = (a0 + a1) + (a2 + a3);
                        }
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < SB; ++q)
                if (have[q] && ok) release(sm, rgs[q]);
        }
        // exchange levels 16 and 8 halve the values a lane holds; levels 4, 2, 1 finish the
        // 32-lane sums: value i ends in lanes 8i..8i+7
        const bool b4 = lane & 16, b3 = lane & 8;
        const float w0 = (b4 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, b4 ? v[0] : v[2], 16);
        const float w1 = (b4 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, b4 ? v[1] : v[3], 16);
        float z = (b3 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, b3 ? w0 : w1, 8);
        z += __shfl_xor_sync(0xffffffffu, z, 4);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        if ((lane & 7) == 0 && ok) {
            const int i = lane >> 3;
            const int js = j0 + i / GM, row = rw + (i % GM) * rstep;
            if (js < nst && row < min(gr, nrows - js * gr)) sm.work[(js * gr + row) * gs + sl] = z;
        }
    }
}

// Dispatch on the chunks per lane and units per warp (fixed per model).
__device__ __forceinline__ void run_rows(const Params& P, const Smem& sm, const unsigned long long* ctl, int nrows,
                                         float scale, Ring& rg, bool& ok, Tracer& tr) {
    const int nch = (P.dm.d >> (__ffs(P.sh.gs) - 1)) >> 8;
    const int gm = P.sh.gm;
    if (gm == 1) {
        switch (nch) {
            case 1: gemv_rows<1, 1>(P, sm, ctl, nrows, scale, rg, ok, tr); break;
            case 2: gemv_rows<2, 1>(P, sm, ctl, nrows, scale, rg, ok, tr); break;
            case 3: gemv_rows<3, 1>(P, sm, ctl, nrows, scale, rg, ok, tr); break;
            default: gemv_rows<4, 1>(P, sm, ctl, nrows, scale, rg, ok, tr); break;
        }
    } else if (gm == 2) {
        gemv_rows<2, 2>(P, sm, ctl, nrows, scale, rg, ok, tr);
    } else {
        gemv_rows<1, 4>(P, sm, ctl, nrows, scale, rg, ok, tr);
    }
}

// Sum of the slices of local row i (after a CTA barrier).
__device__ __forceinline__ float row_value(const Smem& sm, int gs, int i) {
    float v = 0.f;
    for (int s = 0; s < gs; ++s) v += sm.work[i * gs + s];
    return v;
}

// ------------------------------------------------------------------ split-K GEMV

// rows [0, nrows) of a bf16 matrix with rows of d elements (transposed weights: one row per
// input), each scaled by its input value in[row] (shared memory), summed into a d-vector and
// added to `dst` with vector atomics. Thread t owns the outputs of chunk t % (d / 8) (and
// t + 512 when KC == 2) and the rows t / (d / 8) + k * ug of every stage; the ug unit groups
// are summed in shared memory, in group order, before the atomics.
template <int KC>
__device__ __forceinline__ void gemv_splitk(const Params& P, const Smem& sm, const unsigned long long* ctl, int nrows,
                                            const float* in, float* dst, Ring& rg, bool& ok, Tracer& tr) {
    const int d = P.dm.d, oc = d / 8;
    const int kr = P.sh.kr, ug = P.sh.ug;
    const int tid = threadIdx.x;
    const bool active = KC == 2 || tid < ug * oc;
    const int c0 = KC == 2 ? tid : tid % oc, grp = KC == 2 ? 0 : tid / oc;
    const size_t rowbytes = (size_t)d * 2;
    const int nst = (nrows + kr - 1) / kr;
    float acc[KC][8];
#pragma unroll
    for (int c = 0; c < KC; ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[c][e] = 0.f;
    for (int j = 0; j < nst; ++j) {
        if (ok && wait_full(sm, rg, P, ctl, tr.waited)) {
            tr.stage_ready(j, nst);
            const uint8_t* st = sm.ring + (size_t)rg.slot * kStageBytes;
            const int nr = min(kr, nrows - j * kr);
            if (active) {
                for (int row = grp; row < nr; row += ug) {
                    const float a = in[j * kr + row];
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        const int ch = c0 + c * kConsumerThreads;
                        if (KC == 1 || ch < oc) {
                            const uint4 w = lds128(st + row * rowbytes + ch * 16);
                            acc[c][0] = fmaf(bf_lo(w.x), a, acc[c][0]);
                            acc[c][1] = fmaf(bf_hi(w.x), a, acc[c][1]);
                            acc[c][2] = fmaf(bf_lo(w.y), a, acc[c][2]);
                            acc[c][3] = fmaf(bf_hi(w.y), a, acc[c][3]);
                            acc[c][4] = fmaf(bf_lo(w.z), a, acc[c][4]);
                            acc[c][5] = fmaf(bf_hi(w.z), a, acc[c][5]);
                            acc[c][6] = fmaf(bf_lo(w.w), a, acc[c][6]);
                            acc[c][7] = fmaf(bf_hi(w.w), a, acc[c][7]);
                        }
                    }
                }
            }
            release(sm, rg);
        } else {
            ok = false;
        }
        rg.advance(P.ns);
    }
    if (ug > 1) {
        if (active) {
            float4* wp = reinterpret_cast<float4*>(sm.work + (size_t)grp * d + c0 * 8);
            wp[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
            wp[1] = make_float4(acc[0][4], acc[0][5], acc[0][6], acc[0][7]);
        }
        consumer_sync();
        for (int i = tid; i < oc * 2; i += kConsumerThreads) {  // 4 outputs per item
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int g = 0; g < ug; ++g) {
                const float4 v = *reinterpret_cast<const float4*>(sm.work + (size_t)g * d + i * 4);
                s.x += v.x, s.y += v.y, s.z += v.z, s.w += v.w;
            }
            if (ok && nrows > 0) red_add_v4(dst + i * 4, s.x, s.y, s.z, s.w);
        }
    } else if (ok && nrows > 0) {
#pragma unroll
        for (int c = 0; c < KC; ++c) {
            const int ch = c0 + c * kConsumerThreads;
            if (KC == 1 || ch < oc) {
                red_add_v4(dst + ch * 8, acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
                red_add_v4(dst + ch * 8 + 4, acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
            }
        }
    }
}

__device__ __forceinline__ void run_splitk(const Params& P, const Smem& sm, const unsigned long long* ctl, int nrows,
                                           const float* in, float* dst, Ring& rg, bool& ok, Tracer& tr) {
    if (P.sh.kc == 2) gemv_splitk<2>(P, sm, ctl, nrows, in, dst, rg, ok, tr);
    else gemv_splitk<1>(P, sm, ctl, nrows, in, dst, rg, ok, tr);
}

// ------------------------------------------------------------------ phases

// Q/K/V: this CTA's rows of its kv head's block. Row pairs are RoPE pairs (q, k) or
// consecutive dims (v): q is rotated and published; k is rotated, rounded to bf16, appended
// to the cache at position p and published; v is rounded, appended and published.
__device__ __forceinline__ void qkv_epilogue(const Params& P, const Smem& sm, const Geo& g, int l, int p, uint32_t tag) {
    const Dims& dm = P.dm;
    const int hd = dm.hd, r = dm.r, half = hd / 2;
    const int base = g.grp * (r + 2) * hd;
    const int npairs = (g.q1 - g.q0) / 2;
    unsigned long long* out = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.qkv) + base;
    for (int i = threadIdx.x; i < npairs; i += kConsumerThreads) {
        const float a = row_value(sm, P.sh.gs, 2 * i), b = row_value(sm, P.sh.gs, 2 * i + 1);
        const int rr = g.q0 - base + 2 * i;  // row within the kv head's block
        const size_t coff = (((size_t)l * dm.Hkv + g.grp) * dm.S + p) * hd;
        if (rr < (r + 1) * hd) {  // q head or k: RoPE pair (dims j, j + hd/2)
            const int seg = rr / hd, j = (rr % hd) / 2;
            const float2 cs = sm.rope[j];
            float lo = a * cs.x - b * cs.y, hi = b * cs.x + a * cs.y;
            if (seg == r) {  // k: the cache holds bf16
                const __nv_bfloat16 klo = __float2bfloat16_rn(lo), khi = __float2bfloat16_rn(hi);
                __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.kcache) + coff;
                kc[j] = klo, kc[j + half] = khi;
                lo = __bfloat162float(klo), hi = __bfloat162float(khi);
            }
            st_tagged(out + seg * hd + j, lo, tag);
            st_tagged(out + seg * hd + j + half, hi, tag);
        } else {  // v: dims dv, dv + 1
            const int dv = rr - (r + 1) * hd;
            const __nv_bfloat162 v2 = __floats2bfloat162_rn(a, b);
            __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(const_cast<uint8_t*>(P.arena) + P.lay.vcache) + coff;
            *reinterpret_cast<__nv_bfloat162*>(vc + dv) = v2;
            st_tagged(out + (r + 1) * hd + dv, __low2float(v2), tag);
            st_tagged(out + (r + 1) * hd + dv + 1, __high2float(v2), tag);
        }
    }
}

// Attention piece of kv head g at position p (HD: head dim; GM: q heads per kv head
// rounded up to 2, 4 or 8). In each block of cached positions the K stages are scored
// first: a thread takes one position and a quarter of the head dim (32 dims, its q slices
// held in registers, two q heads per pass), the quarters are summed in shared memory in
// quarter order, and the block's max and exponentials are formed once; the V stages then
// accumulate with thread (dim pair, position group) ownership. Blocks after the first
// rescale the running state once. The piece publishes one record per q head: the running
// max (log2 domain), the sum of exponentials and the unnormalised output.
template <int HD, int GM>
__device__ __forceinline__ void run_attention(const Params& P, const Smem& sm, const unsigned long long* ctl, int t, int l,
                                              Ring& rg, bool& ok, Tracer& tr) {
    const Dims& dm = P.dm;
    const Geo& g = *sm.geo;
    const int r = dm.r;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p = P.pos0 + t;
    const Piece pc = *sm.piece;
    const uint32_t tag = qkv_tag(P, t, l);
    constexpr int PPS = kStageBytes / (2 * HD);     // positions per stage
    constexpr int NQ = HD / 32;                     // quarters of the head dim (32 dims each)
    constexpr int WPQ = kConsumerWarps / NQ;        // warps per quarter
    constexpr int NPG = kConsumerThreads / (HD / 2);  // V position groups
    constexpr int RP = GM;                          // score row stride (heads, padded)
    float* sc = sm.work;                            // [blk + 1][RP] scores, then probabilities
    float* spart = sm.work + (size_t)(P.blk + 1) * RP;  // [2][NQ][GM][PPS] quarter partials
    float* vred = spart;                            // [NPG][GM][HD] at the end

    // ---- inputs: q of the group's heads (prescaled for exp2), and the current k / v
    {
        const unsigned long long* src =
            reinterpret_cast<const unsigned long long*>(P.arena + P.lay.qkv) + (size_t)g.grp * (r + 2) * HD;
        const int nq = r * HD, nw = pc.cur ? nq + 2 * HD : nq;
        const float qscale = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
        unsigned long long w[3];
#pragma unroll
        for (int u = 0; u < 3; ++u)
            if (tid + u * kConsumerThreads < nw) w[u] = ld_tagged(src + tid + u * kConsumerThreads);
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const int i = tid + u * kConsumerThreads;
            if (i < nw) {
                if (!get_word(src + i, tag, w[u], P, ctl, 3)) ok = false;
                const float v = tagged_value(w[u]);
                if (i < nq) sm.qs[i] = v * qscale;
                else sm.kvc[i - nq] = v;
            }
        }
    }
    ok = consumer_sync_and(ok);  // every thread's words (a failed poll stops the whole CTA)
    tr.mark(2);

    // score-pass ownership: quarter qq, position j of a stage
    const int qq = warp / WPQ;
    const int jpos = (warp % WPQ) * 32 + lane;
    // V-pass ownership: dims 2 dp, 2 dp + 1, positions pg, pg + NPG, ...
    const int dp = tid % (HD / 2), pg = tid / (HD / 2);
    // running max (log2 domain) and sum per head live in shared memory (stats[h], stats[GM + h]):
    // every thread would hold the same values, and registers are short here
    float acc[GM][2];
#pragma unroll
    for (int h = 0; h < GM; ++h) acc[h][0] = acc[h][1] = 0.f;
    if (tid < GM) sm.stats[tid] = -INFINITY, sm.stats[GM + tid] = 0.f;
    for (int kb = 0; kb < pc.nblk; ++kb) {
        const int n = block_len(P, pc, kb);
        const bool last = kb == pc.nblk - 1;
        const bool with_cur = pc.cur && last;
        const int nks = (n + PPS - 1) / PPS;
        // ---- K stages: scores
        for (int js = 0; js < nks; ++js) {
            float* sp = spart + (size_t)(js & 1) * NQ * GM * PPS;
            if (ok && wait_full(sm, rg, P, ctl, tr.waited)) {
                if (kb == 0 && js == 0) tr.mark(6);
                const uint8_t* st = sm.ring + (size_t)rg.slot * kStageBytes;
                const int nv = min(PPS, n - js * PPS);
                // chunk c of this thread's quarter is taken in a rotated order (c + jpos) & 3,
                // so the lanes of a quarter-warp read different bank groups of their K rows;
                // q is read from shared memory at the same rotated chunk (four addresses per
                // warp, one per rotation, each broadcast)
                float sh[GM];
#pragma unroll
                for (int h = 0; h < GM; ++h) sh[h] = 0.f;
                if (jpos < nv) {
                    const uint8_t* krow = st + (size_t)jpos * HD * 2 + qq * 64;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int cc = (c + jpos) & 3;
                        const uint4 w = lds128(krow + cc * 16);
                        const float k0 = bf_lo(w.x), k1 = bf_hi(w.x), k2 = bf_lo(w.y), k3 = bf_hi(w.y);
                        const float k4 = bf_lo(w.z), k5 = bf_hi(w.z), k6 = bf_lo(w.w), k7 = bf_hi(w.w);
#pragma unroll
                        for (int h = 0; h < GM; ++h) {
                            if (h < r) {
                                const float* q = sm.qs + (size_t)h * HD + qq * 32 + cc * 8;
                                const float4 qa = *reinterpret_cast<const float4*>(q);
                                const float4 qb = *reinterpret_cast<const float4*>(q + 4);
                                float t = sh[h];
                                t = fmaf(k0, qa.x, t), t = fmaf(k1, qa.y, t), t = fmaf(k2, qa.z, t), t = fmaf(k3, qa.w, t);
                                t = fmaf(k4, qb.x, t), t = fmaf(k5, qb.y, t), t = fmaf(k6, qb.z, t), t = fmaf(k7, qb.w, t);
                                sh[h] = t;
                            }
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < GM; ++h) sp[((size_t)qq * GM + h) * PPS + jpos] = sh[h];
                release(sm, rg);
            } else {
                ok = false;
            }
            rg.advance(P.ns);
            consumer_sync();  // the quarter partials of stage js are complete
            const int nv = min(PPS, n - js * PPS);
            for (int i = tid; i < nv * GM; i += kConsumerThreads) {
                const int j = i / GM, h = i % GM;
                float s = 0.f;
#pragma unroll
                for (int q = 0; q < NQ; ++q) s += sp[((size_t)q * GM + h) * PPS + j];
                sc[(size_t)(js * PPS + j) * RP + h] = s;
            }
        }
        // the current position's scores (warp h, HD / 32 dims per lane)
        if (with_cur && warp < r) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < HD / 32; ++e) s = fmaf(sm.qs[warp * HD + lane * (HD / 32) + e], sm.kvc[lane * (HD / 32) + e], s);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) sc[(size_t)n * RP + warp] = s;
        }
        consumer_sync();  // all scores of the block
        // ---- block softmax statistics: max, then exponentials and their sum
        const int ns_ = n + (with_cur ? 1 : 0);
        float mx[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) mx[h] = -INFINITY;
        for (int j = tid; j < ns_; j += kConsumerThreads)
#pragma unroll
            for (int h = 0; h < GM; ++h)
                if (h < r) mx[h] = fmaxf(mx[h], sc[(size_t)j * RP + h]);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
            if (lane == 0 && h < 8) sm.red[warp * 8 + h] = mx[h];
        }
        consumer_sync();
        float mnew[GM], corr[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            const float mold = sm.stats[h];
            float m = mold;
            if (h < r)
                for (int w = 0; w < kConsumerWarps; ++w) m = fmaxf(m, sm.red[w * 8 + h]);
            mnew[h] = m;
            corr[h] = m == -INFINITY ? 0.f : exp2f(mold - m);  // no positions yet: nothing to rescale
        }
        consumer_sync();  // red and stats are rewritten below
        float ls[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) ls[h] = 0.f;
        for (int j = tid; j < ns_; j += kConsumerThreads)
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                const float e = h < r ? exp2f(sc[(size_t)j * RP + h] - mnew[h]) : 0.f;
                sc[(size_t)j * RP + h] = e;
                ls[h] += e;
            }
#pragma unroll
        for (int h = 0; h < GM; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], o);
            if (lane == 0 && h < 8) sm.red[warp * 8 + h] = ls[h];
            acc[h][0] *= corr[h];
            acc[h][1] *= corr[h];
        }
        consumer_sync();  // probabilities and partial sums complete
        if (tid < GM) {
            float s = 0.f;
            for (int w = 0; w < kConsumerWarps; ++w) s += sm.red[w * 8 + tid];
            float cr = 0.f, mn = 0.f;
#pragma unroll
            for (int h = 0; h < GM; ++h)
                if (h == tid) cr = corr[h], mn = mnew[h];
            sm.stats[GM + tid] = sm.stats[GM + tid] * cr + s;
            sm.stats[tid] = mn;
        }
        // ---- V stages
        for (int js = 0; js < nks; ++js) {
            if (ok && wait_full(sm, rg, P, ctl, tr.waited)) {
                if (last && js == nks - 1) tr.mark(7);
                const uint8_t* st = sm.ring + (size_t)rg.slot * kStageBytes;
                const int nv = min(PPS, n - js * PPS);
                for (int j = pg; j < nv; j += NPG) {
                    const uint32_t vw = *reinterpret_cast<const uint32_t*>(st + (size_t)j * HD * 2 + dp * 4);
                    const float v0 = bf_lo(vw), v1 = bf_hi(vw);
                    const float* pr = sc + (size_t)(js * PPS + j) * RP;
                    float pv[GM];
                    if constexpr (GM == 2) {
                        const float2 a = *reinterpret_cast<const float2*>(pr);
                        pv[0] = a.x, pv[1] = a.y;
                    } else {
#pragma unroll
                        for (int h4 = 0; h4 < GM; h4 += 4) {
                            const float4 a = *reinterpret_cast<const float4*>(pr + h4);
                            pv[h4] = a.x, pv[h4 + 1] = a.y, pv[h4 + 2] = a.z, pv[h4 + 3] = a.w;
                        }
                    }
#pragma unroll
                    for (int h = 0; h < GM; ++h) {
                        acc[h][0] = fmaf(pv[h], v0, acc[h][0]);
                        acc[h][1] = fmaf(pv[h], v1, acc[h][1]);
                    }
                }
                release(sm, rg);
            } else {
                ok = false;
            }
            rg.advance(P.ns);
        }
        if (with_cur && pg == 0) {
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                const float pcur = h < r ? sc[(size_t)n * RP + h] : 0.f;
                acc[h][0] = fmaf(pcur, sm.kvc[HD + 2 * dp], acc[h][0]);
                acc[h][1] = fmaf(pcur, sm.kvc[HD + 2 * dp + 1], acc[h][1]);
            }
        }
        consumer_sync();  // scores, probabilities and red are reused by the next block
    }
    tr.mark(3);
    // ---- record: sum the position groups in group order, publish (max, sum, acc)
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h < r) {
            float2* vp = reinterpret_cast<float2*>(vred + ((size_t)pg * GM + h) * HD + 2 * dp);
            *vp = make_float2(acc[h][0], acc[h][1]);
        }
    }
    consumer_sync();
    unsigned long long* rec = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.rec) +
                              (size_t)blockIdx.x * r * (HD + 2);
    for (int i = tid; i < r * HD; i += kConsumerThreads) {
        const int h = i / HD, dd = i % HD;
        float s = 0.f;
        for (int q = 0; q < NPG; ++q) s += vred[((size_t)q * GM + h) * HD + dd];
        st_tagged(rec + (size_t)h * (HD + 2) + 2 + dd, s, tag + 1u);
    }
    if (tid < r) {
        st_tagged(rec + (size_t)tid * (HD + 2), sm.stats[tid], tag + 1u);
        st_tagged(rec + (size_t)tid * (HD + 2) + 1, sm.stats[GM + tid], tag + 1u);
    }
}

// Output-projection inputs: combine the attention records of every piece of this CTA's kv
// head for its own output dims (max-rescaled sums over the pieces) into sm.hin. Returns the
// number of dims (rows of the transposed output projection this CTA multiplies).
template <int HD>
__device__ __forceinline__ int oproj_inputs(const Params& P, const Smem& sm, const unsigned long long* ctl, int t, int l,
                                            bool& ok, Tracer& tr) {
    const Dims& dm = P.dm;
    const Geo& g = *sm.geo;
    const int r = dm.r, A = P.pieces;
    const int cc = r * HD;
    const int c0 = g.o0 - g.grp * cc, c1 = g.o1 - g.grp * cc;  // dims within the kv head's heads
    const int ncol = c1 - c0;
    if (ncol <= 0) return 0;  // more pieces than output dims: this CTA has none (uniform)
    const int h0 = c0 / HD, h1 = (c1 - 1) / HD, nh = h1 - h0 + 1;
    const int W = 2 * nh + ncol;  // words per piece: (max, sum) per head, then acc per dim
    const uint32_t tag = qkv_tag(P, t, l) + 1u;
    const unsigned long long* rec = reinterpret_cast<const unsigned long long*>(P.arena + P.lay.rec);
    float* stage = sm.work;  // [A][W]
    for (int i = threadIdx.x; i < A * W; i += kConsumerThreads) {
        const int pi = i / W, k = i % W;
        const int cta = g.grp * A + pi;
        int h, word;
        if (k < 2 * nh) {
            h = h0 + k / 2;
            word = k & 1;
        } else {
            const int col = c0 + k - 2 * nh;
            h = col / HD;
            word = 2 + col % HD;
        }
        const unsigned long long* src = rec + ((size_t)cta * r + h) * (HD + 2) + word;
        unsigned long long w = ld_tagged(src);
        if (!get_word(src, tag, w, P, ctl, 5)) ok = false;
        stage[i] = tagged_value(w);
    }
    ok = consumer_sync_and(ok);
    tr.mark(2);
    // one warp per output dim, its lanes over the pieces; the max and the two sums are
    // reduced across the warp (a fixed shuffle tree)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = warp; j < ncol; j += kConsumerWarps) {
        const int col = c0 + j, hi = col / HD - h0;
        float M = -INFINITY;
        for (int pi = lane; pi < A; pi += 32) M = fmaxf(M, stage[pi * W + 2 * hi]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f, o = 0.f;
        for (int pi = lane; pi < A; pi += 32) {
            const float f = exp2f(stage[pi * W + 2 * hi] - M);  // 0 for an empty piece
            L = fmaf(stage[pi * W + 2 * hi + 1], f, L);
            o = fmaf(stage[pi * W + 2 * nh + j], f, o);
        }
#pragma unroll
        for (int s2 = 16; s2 > 0; s2 >>= 1) {
            L += __shfl_xor_sync(0xffffffffu, L, s2);
            o += __shfl_xor_sync(0xffffffffu, o, s2);
        }
        if (lane == 0) sm.hin[j] = o / L;
    }
    consumer_sync();
    return ncol;
}

// ------------------------------------------------------------------ producer

// Walks this CTA's stages in consumption order: per step, per layer the Q/K/V rows, the
// attention piece (per softmax block its K stages, then its V stages), the output-projection
// rows, the gate/up rows, the down-projection rows; then the LM-head rows at steps that run
// the head. Sub-phase `sub` of a layer: 0 Q/K/V, 1 .. 2 * nblk attention (block (sub - 1) / 2,
// K for odd sub, V for even), then output projection, gate/up, down, and after the last layer
// the LM head.
struct Walk {
    int t = 0, l = 0, sub = 0, j = 0;
    int pc_t = -1;
    Piece pc;
    bool done = false;

    // The current sub-phase's rows: base, bytes per row, rows, rows per stage, and the first
    // cache position (-1 for weights).
    __device__ void desc(const Params& P, const Geo& g, const uint8_t*& base, size_t& rowb, int& nrows, int& per,
                         int& pos) {
        const Dims& dm = P.dm;
        const size_t wrow = (size_t)dm.d * 2;
        const uint8_t* lb = P.arena + P.lay.layer0 + (size_t)l * P.lay.layer_stride;
        const int natt = g.grp < 0 ? 0 : 2 * pc.nblk;
        pos = -1;
        rowb = wrow;
        if (sub == 0) {
            base = lb + P.lay.l_wqkv + (size_t)g.q0 * wrow, nrows = g.q1 - g.q0, per = P.sh.gr;
        } else if (sub <= natt) {
            const int kb = (sub - 1) / 2;
            const int s0 = pc.a + kb * P.blk;
            const size_t head = ((size_t)l * dm.Hkv + g.grp) * dm.S;
            rowb = (size_t)dm.hd * 2;
            base = P.arena + ((sub & 1) ? P.lay.kcache : P.lay.vcache) + (head + s0) * rowb;
            nrows = block_len(P, pc, kb), per = kStageBytes / (int)rowb, pos = s0;
        } else if (sub == natt + 1) {
            base = lb + P.lay.l_wot + (size_t)g.o0 * wrow, nrows = g.o1 - g.o0, per = P.sh.kr;
        } else if (sub == natt + 2) {
            base = lb + P.lay.l_wgu + (size_t)2 * g.u0 * wrow, nrows = 2 * (g.u1 - g.u0), per = P.sh.gr;
        } else if (sub == natt + 3) {
            base = lb + P.lay.l_wdt + (size_t)g.u0 * wrow, nrows = g.u1 - g.u0, per = P.sh.kr;
        } else {
            base = P.arena + P.lay.lm_head + (size_t)g.v0 * wrow, nrows = g.v1 - g.v0, per = P.sh.gr;
        }
    }
    __device__ int nsubs(const Params& P, const Geo& g) const {
        const int natt = g.grp < 0 ? 0 : 2 * pc.nblk;
        return natt + 4 + (l == P.dm.L - 1 && step_has_head(P, t) ? 1 : 0);
    }
    // The next stage: source, bytes, and the last cache position it reads (-1 for weights).
    // Returns false when the launch's stages are exhausted.
    __device__ bool next(const Params& P, const Geo& g, const uint8_t*& src, uint32_t& bytes, int& kv_last) {
        for (;;) {
            if (done) return false;
            if (pc_t != t) {
                pc = piece_geo(P, g.piece, P.pos0 + t);
                pc_t = t;
            }
            const uint8_t* base;
            size_t rowb;
            int nrows, per, pos;
            desc(P, g, base, rowb, nrows, per, pos);
            if (j * per < nrows) {
                const int n = min(per, nrows - j * per);
                src = base + (size_t)j * per * rowb;
                bytes = (uint32_t)(n * rowb);
                kv_last = pos < 0 ? -1 : pos + j * per + n - 1;
                ++j;
                return true;
            }
            j = 0;
            if (++sub >= nsubs(P, g)) {
                sub = 0;
                if (++l == P.dm.L) {
                    l = 0;
                    if (++t == P.steps) done = true;
                }
            }
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
    long long seen = 0;      // syncs known complete
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
        const long long c0 = clock64();
        Deadline dl;
        for (;;) {
            if (mbar_wait_hint(a, par)) break;
            if (!dl.alive(ctl, P.timeout_ns, where_code(kWhereEmpty, slot))) return false;
        }
        wait_slot += (unsigned long long)(clock64() - c0);
        return true;
    }

    // Wait until at least `need` syncs of this launch have completed, then order the
    // generic-proxy cache writes they publish before this thread's later bulk copies.
    __device__ bool wait_syncs(long long need) {
        if (seen >= need) return true;
        const long long c0 = clock64();
        Deadline dl;
        for (uint32_t it = 0;; ++it) {
            seen = (long long)((ld_acquire_u64(reinterpret_cast<const unsigned long long*>(sm.u64[1])) - base) /
                               (uint64_t)P.nb);
            if (seen >= need) break;
            if ((it & 31) == 31 && !dl.alive(ctl, P.timeout_ns, where_code(kWhereKv, 0))) return false;
        }
        wait_kv += (unsigned long long)(clock64() - c0);
        fence_proxy_async_global();
        return true;
    }

    // Stage k into its ring slot. A cache row written earlier in this launch (at step s) is
    // read only after the last sync of step s, which orders that step's cache writes.
    __device__ bool issue(const uint8_t* src, uint32_t bytes, int kv_last) {
        if (kv_last >= P.pos0) {
            const int s = kv_last - P.pos0;
            if (!wait_syncs(syncs_before_step(P.dm.L, s + 1, P.n_pending, P.dump != 0))) return false;
        }
        if (!wait_empty()) return false;
        const uint32_t fb = smem_u32(&sm.full[slot]);
        mbar_expect_tx(fb, bytes);
        bulk_g2s(smem_u32(sm.ring + (size_t)slot * kStageBytes), src, bytes, fb, policy);
        ++k;
        if (++slot == P.ns) {
            slot = 0;
            ++pass;
        }
        return true;
    }

    __device__ void run() {
        const long long c_start = clock64();
        const Geo g = *sm.geo;
        Walk ring;
        const uint8_t* src;
        uint32_t bytes;
        int kv_last;
        bool ok = true;
        while (ok && ring.next(P, g, src, bytes, kv_last)) ok = issue(src, bytes, kv_last);
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
            unsigned long long* r =
                P.trace + ((size_t)(blockIdx.x / P.trace_every) * P.trace_rows + P.trace_rows - 1) * kTraceWords;
            r[0] = wait_slot, r[1] = wait_kv, r[2] = (unsigned long long)k;
            r[3] = (unsigned long long)(clock64() - c_start);
        }
    }
};

// ------------------------------------------------------------------ the kernel

// ---- temperature sampling: the Gumbel-max draw from softmax(logits / T)
//
// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC 2011): a 128-bit counter, a 64-bit key, ten rounds of two 32x32 -> 64-bit products, the
// key bumped between rounds by the two Weyl constants.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) k0 += 0x9E3779B9u, k1 += 0xBB67AE85u;
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    }
    return c;
}
// logit * (1/T) + g for vocabulary index i at absolute position pos, g = -log(-log(u)) with u
// the (i mod 4)-th word of Philox((i div 4, pos, 0, 0), seed): its top 23 bits + 0.5, / 2^23
// (exact in fp32, so u is never 0 or 1).
__device__ __forceinline__ float gumbel_perturbed(const Params& P, float y, int i, int pos) {
    const uint4 w = philox4x32_10(make_uint4((uint32_t)i >> 2, (uint32_t)pos, 0u, 0u), P.seed_lo, P.seed_hi);
    const int q = i & 3;
    const uint32_t x = q == 0 ? w.x : q == 1 ? w.y : q == 2 ? w.z : w.w;
    const float u = ((float)(x >> 9) + 0.5f) * 1.1920928955078125e-7f;  // 2^-23
    return y * P.inv_temp - logf(-logf(u));
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xffffffffu - (uint32_t)idx);
}
__device__ __forceinline__ int key_index(unsigned long long key) {
    return (int)(0xffffffffu - (uint32_t)(key & 0xffffffffull));
}

// One instantiation per attention shape (head dim, q heads per kv head rounded up to 2, 4
// or 8), so the fully inlined kernel holds one attention body and its registers.
template <int HD, int GM>
__global__ void __launch_bounds__(kThreads, 1) monokernel(const __grid_constant__ Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem sm = carve(P, smem_raw);
    unsigned long long* ctl = reinterpret_cast<unsigned long long*>(const_cast<uint8_t*>(P.arena) + P.lay.ctl);
    const int tid = threadIdx.x;
    const Dims& dm = P.dm;

    if (tid == 0) {
        for (int s = 0; s < P.ns; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), kConsumerWarps);  // every consumer warp releases every stage
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        cta_geo(P, blockIdx.x, *sm.geo);
        // The counter replica local to this SM (kd_create measured which die owns which), and
        // the other one if there are two.
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        const int rep = P.nsync == 2 && smid < (uint32_t)kMaxSmid ? (P.arena[P.lay.dietab + smid] & 1) : 0;
        uint8_t* ab = const_cast<uint8_t*>(P.arena);
        sm.u64[1] = reinterpret_cast<unsigned long long>(ab + P.sync_off[rep]);
        sm.u64[2] = P.nsync == 2 ? reinterpret_cast<unsigned long long>(ab + P.sync_off[rep ^ 1]) : 0ull;
        // Sync count at launch: a multiple of nb (every launch that completed arrived nb times
        // at each of its syncs, on every replica) plus arrivals of CTAs already at this launch's
        // first sync (which cannot complete before this CTA arrives).
        const uint64_t raw = ld_acquire_u64(reinterpret_cast<const unsigned long long*>(sm.u64[1]));
        sm.u64[0] = raw - raw % (uint64_t)P.nb;
        sm.flag[0] = read_status(ctl);
    }
    __syncthreads();
    const uint64_t base = sm.u64[0];
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
    const Geo& g = *sm.geo;
    int32_t* tokens_in = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(P.arena) + P.lay.tokens_in);
    const __nv_bfloat16* embed = reinterpret_cast<const __nv_bfloat16*>(P.arena + P.lay.embed);
    float* delta = reinterpret_cast<float*>(const_cast<uint8_t*>(P.arena) + P.lay.delta);
    const uint8_t* l0 = P.arena + P.lay.layer0;
    Ring rg;
    bool ok = true;
    Tracer tr;
    if (P.trace && tid == 0 && blockIdx.x % P.trace_every == 0) {
        tr.row0 = P.trace + (size_t)(blockIdx.x / P.trace_every) * P.trace_rows * kTraceWords;
        tr.rows = P.trace_rows;
    }
    long long k = 0;  // syncs of this launch so far (the next one to arrive at)

    for (int t = 0; t < P.steps && ok; ++t) {
        const int p = P.pos0 + t;
        // ---- token: a pending input, or the argmax of the previous step
        if (t > 0) {
            ok = sync_wait(sm, P, ctl, k - 1, ok);
            if (!ok) break;
        }
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
            if (g.grp >= 0) *sm.piece = piece_geo(P, g.piece, p);  // 64-bit divisions, once per step
        }
        if (tid < dm.hd / 2)  // this position's RoPE row (cos, sin per pair)
            sm.rope[tid] = __ldg(reinterpret_cast<const float2*>(P.arena + P.lay.rope) + (size_t)p * (dm.hd / 2) + tid);
        consumer_sync();
        const int tok = sm.flag[2];
        if (tok < 0) {
            ok = false;
            break;
        }
        if (t > 0) zero_previous(P, k - 1);
        {
            const __nv_bfloat16* erow = embed + (size_t)tok * dm.d;
            for (int i = tid * 4; i < dm.d; i += kConsumerThreads * 4) {
                const uint2 e = __ldg(reinterpret_cast<const uint2*>(erow + i));
                *reinterpret_cast<float4*>(sm.x + i) = make_float4(bf_lo(e.x), bf_hi(e.x), bf_lo(e.y), bf_hi(e.y));
            }
        }
        consumer_sync();

        // The step's phases in order: per layer Q/K/V, attention, output projection, gate/up,
        // down; then the LM head if this step picks a token. One loop with one call site per
        // phase kind keeps a single copy of each phase's code in the kernel (the executed
        // code then stays in the instruction cache across layers).
        const int nphase = 5 * dm.L + (step_has_head(P, t) ? 1 : 0);
        for (int q = 0; q < nphase && ok; ++q) {
            const int l = q / 5 < dm.L ? q / 5 : dm.L - 1;
            const int ph = q / 5 < dm.L ? q % 5 : kLM;
            const uint8_t* lb = l0 + (size_t)l * P.lay.layer_stride;
            tr.begin((t << 16) | (l << 4) | ph);
            if (ph == kQKV || ph == kGU || ph == kLM) {
                // ---- row GEMV: Q/K/V, gate/up or LM head over the normalised residual
                const uint8_t* gain = ph == kQKV ? lb + P.lay.l_attn_norm
                                      : ph == kGU ? lb + P.lay.l_ffn_norm : P.arena + P.lay.final_norm;
                prefetch_gain(sm, reinterpret_cast<const __nv_bfloat16*>(gain), dm.d);
                const bool after_sync = !(ph == kQKV && l == 0);  // the first Q/K/V reads the embedding
                if (after_sync) {
                    ok = sync_wait(sm, P, ctl, k - 1, ok);
                    if (!ok) break;
                }
                const float s = fold_norm(sm, P, after_sync ? k - 1 : -1);
                tr.mark(2);
                const int nrows = ph == kQKV ? g.q1 - g.q0 : ph == kGU ? 2 * (g.u1 - g.u0) : g.v1 - g.v0;
                run_rows(P, sm, ctl, nrows, s, rg, ok, tr);
                ok = consumer_sync_and(ok);
                if (ph == kQKV) {
                    tr.mark(3);
                    if (ok && g.grp >= 0) qkv_epilogue(P, sm, g, l, p, qkv_tag(P, t, l));
                } else if (ph == kGU) {
                    for (int j = tid; j < g.u1 - g.u0; j += kConsumerThreads) {
                        const float gt = row_value(sm, P.sh.gs, 2 * j), up = row_value(sm, P.sh.gs, 2 * j + 1);
                        sm.hin[j] = gt / (1.0f + expf(-gt)) * up;
                    }
                    ok = consumer_sync_and(ok);
                    tr.mark(3);
                } else {
                    unsigned long long best = 0ull;
                    for (int i = tid; i < g.v1 - g.v0; i += kConsumerThreads) {
                        const float y = row_value(sm, P.sh.gs, i);
                        if (P.dump) __stcg(P.logits_out + (size_t)t * dm.V + g.v0 + i, y);
                        const float z = P.inv_temp > 0.f ? gumbel_perturbed(P, y, g.v0 + i, p) : y;
                        const unsigned long long key = argmax_key(z, g.v0 + i);
                        best = key > best ? key : best;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
                        best = other > best ? other : best;
                    }
                    if ((tid & 31) == 0) reinterpret_cast<unsigned long long*>(sm.red)[tid >> 5] = best;
                    ok = consumer_sync_and(ok);
                    if (tid == 0 && ok) {
                        unsigned long long b = 0ull;
                        for (int w = 0; w < kConsumerWarps; ++w) {
                            const unsigned long long v = reinterpret_cast<unsigned long long*>(sm.red)[w];
                            b = v > b ? v : b;
                        }
                        red_max_u64(ctl + kCtlArgmax + 16 * (t % 3), b);
                    }
                    tr.mark(3);
                    if (ok) sync_arrive(sm);  // -> sync k: the step's argmax is complete
                    ++k;
                }
            } else if (ph == kATT) {
                // ---- attention piece
                if (g.grp >= 0) run_attention<HD, GM>(P, sm, ctl, t, l, rg, ok, tr);
                ok = consumer_sync_and(ok);
            } else {
                // ---- split-K output projection or down projection -> sync k
                tr.mark(2);
                int nrows = g.u1 - g.u0;  // down: this CTA's hidden units (sm.hin, from gate/up)
                if (ph == kO) nrows = g.grp >= 0 ? oproj_inputs<HD>(P, sm, ctl, t, l, ok, tr) : 0;
                run_splitk(P, sm, ctl, nrows, sm.hin,
                           delta + ((size_t)(k % 3) * kSumCopies + blockIdx.x % kSumCopies) * dm.d, rg, ok, tr);
                tr.mark(3);
                ok = consumer_sync_and(ok);
                if (ok) sync_arrive(sm);
                ++k;
            }
            tr.end();
        }
    }
    if (ok && k > 0) {
        // Wait for the launch's last sync, then leave all three delta buffers zero for the next
        // launch: the one of the second-to-last sync is zeroed here like at every wait, and
        // the last one (read by nobody after the launch) too.
        ok = sync_wait(sm, P, ctl, k - 1, ok);
        if (ok) {
            const int n = kSumCopies * dm.d;  // a buffer with all its copies
            const int z0 = (int)((long long)n * blockIdx.x / P.nb), z1 = (int)((long long)n * (blockIdx.x + 1) / P.nb);
            for (int i = z0 + tid; i < z1; i += kConsumerThreads) {
                delta[(size_t)((k - 1) % 3) * n + i] = 0.f;
                if (k >= 2) delta[(size_t)((k - 2) % 3) * n + i] = 0.f;
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
        // every CTA has read the earlier slots; the next launch starts from cleared ones
        for (int s = 0; s < 3; ++s) ctl[kCtlArgmax + 16 * s] = 0ull;
    }
}

// ------------------------------------------------------------------ host-side launch

static const void* kernel_for(const Dims& dm) {
    if (dm.hd == 128) {
        if (dm.r <= 2) return (const void*)monokernel<128, 2>;
        if (dm.r <= 4) return (const void*)monokernel<128, 4>;
        return (const void*)monokernel<128, 8>;
    }
    if (dm.r <= 2) return (const void*)monokernel<64, 2>;
    if (dm.r <= 4) return (const void*)monokernel<64, 4>;
    return (const void*)monokernel<64, 8>;
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
