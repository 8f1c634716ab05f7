// kd_layout.h -- arena layout, launch constants and kernel parameters shared by the host
// side of libkd (kd_api.cu) and the monokernel (kd_kernel.cu). Internal to libkd.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace kd {

// Pipeline: one producer warp streams weight / KV tiles into a ring of shared-memory
// stages with 1-D bulk copies; consumer warps each take whole stages round-robin.
constexpr int kStageBytes = 32768;
constexpr int kGroupWarps = 8;                      // warps that share one pipeline stage
constexpr int kGroups = 1;                          // groups take alternate stages (slot parity)
constexpr int kConsumerWarps = kGroupWarps * kGroups;  // + 1 producer warp
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxRows = 8;       // rows of one GEMV stage (one per warp of a group)
constexpr int kMaxChunks = 8;     // 16-byte weight chunks per lane per row slice (x kept in registers)
constexpr int kMaxGroup = 8;      // q heads per kv head
constexpr int kMaxKvHeads = 16;
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;  // opt-in dynamic shared memory per CTA on B200

// Control words (uint64), each on its own 128-byte line.
constexpr int kCtlBar = 0;                 // grid-barrier arrivals, monotonic
constexpr int kCtlStatus = 16;             // 0 = ok, else an error code (device side)
constexpr int kCtlWhere = 17;              // where a wait gave up (debug)
constexpr int kCtlArgmax = 32;             // 3 argmax slots at kCtlArgmax + 16*i
constexpr int kCtlHead = 96;               // split-K arrival counters at kCtlHead + 16*g
constexpr int kCtlWords = kCtlHead + 16 * kMaxKvHeads;

constexpr int kStatusTimeout = 1;  // a device-side wait exceeded its limit
constexpr int kStatusToken = 2;    // a token id outside [0, vocab) reached the kernel

struct Dims {
    int L, d, Hq, Hkv, hd, F, V, S;  // S = max_seq
    float eps, theta;
    int qd, kvd, r;  // Hq*hd, Hkv*hd, Hq/Hkv
    int qkv_rows;    // (Hq + 2*Hkv) * hd
};

// Byte offsets inside the arena.
struct Layout {
    size_t embed, lm_head, final_norm;
    size_t layer0, layer_stride;
    size_t l_attn_norm, l_ffn_norm, l_wqkv, l_wo, l_wgu, l_wd;  // within a layer block
    size_t rope;                                                  // [S][hd/2] float2 (cos, sin)
    size_t kcache, vcache;                                        // [L][Hkv][S][hd] bf16
    // Activations exchanged between CTAs, each element a 64-bit word (fp32 value in the low
    // half, the producing phase's tag in the high half): x [2][d] (outputs of O and of D),
    // qkv [qkv_rows], o [qd], gu [F] (the FFN hidden vector). Attention partials are fp32.
    size_t x, qkv, o, gu, part;
    size_t ctl, tokens_in, tokens_out;
    size_t weights_end, kv_bytes, total;
};

// Rows per pipeline stage of one GEMV phase with reduction length K (bf16 elements): the
// largest power of two <= 8 whose rows fit a stage. The kernel cuts each row into slices
// (16 / R of them when R >= 2, else 8) shared by the 8 consumer warps.
inline int rows_per_stage(int K, bool paired) {
    int r = kStageBytes / (2 * K);
    if (r > kMaxRows) r = kMaxRows;
    int p2 = 1;
    while (p2 * 2 <= r) p2 *= 2;
    (void)paired;
    return p2;
}

// Chunks of 8 elements per lane that a GEMV slice of reduction length K needs when a stage
// holds R = rows_per_stage(K) rows cut into 16 / R slices (R >= 2) or 8 slices (R == 1).
inline int gemv_slice_chunks(int K) {
    const int R = rows_per_stage(K, false);
    const int slices = R >= 2 ? 16 / R : 8;
    return (K / slices + 255) / 256;
}
inline int gemv_max_chunks(const Dims& dm) {
    int m = gemv_slice_chunks(dm.d);
    if (gemv_slice_chunks(dm.qd) > m) m = gemv_slice_chunks(dm.qd);
    if (gemv_slice_chunks(dm.F) > m) m = gemv_slice_chunks(dm.F);
    return m;
}

// Phases one launch runs: per step 5 per layer (QKV, ATT, O, GU, D), plus the LM head at
// the steps that pick a token (or at every step when logits are dumped). Tags of
// successive launches follow each other, so a buffer element never carries a stale tag
// that a reader of a later launch expects.
inline long long launch_phases(const Dims& dm, int steps, int n_pending, bool dump) {
    const long long heads = dump ? steps : (steps - (n_pending - 1) > 0 ? steps - (n_pending - 1) : 0);
    return (long long)steps * 5 * dm.L + heads;
}

struct Params {
    // weights (arena)
    const uint8_t* arena;
    Layout lay;
    Dims dm;
    // per-launch
    int steps;      // decode steps in this launch
    int n_pending;  // tokens fed before the first generated one
    int pos0;       // position of step 0
    int n_gen;
    int dump;       // write logits of every step
    int32_t* tokens_out;
    float* logits_out;
    // launch shape
    int nb;           // CTAs
    int ns;           // pipeline stages
    int attn_pieces;  // CTAs per kv head in attention
    int pos_per_stage;
    int rows_qkv, rows_o, rows_gu, rows_d, rows_lm;  // rows per stage of each GEMV phase
    int xs_floats;                                    // activation buffer (floats)
    int xown_floats;                                  // this CTA's residual rows (floats)
    long long timeout_ns;
    int prefetch;  // stages the producer pulls into L2 ahead of the shared-memory ring
    int inflight;  // at most this many issued stages not yet landed (bounds memory queueing)
    uint32_t tag0;  // phase i of this launch tags its outputs tag0 + 1 + i (see kd_kernel.cu)
    // optional trace: CTAs with blockIdx.x % trace_every == 0 record per-phase timestamps
    unsigned long long* trace;
    int trace_every, trace_rows;  // rows per traced CTA (4 words each)
};

// Trace row layout (SM clock cycles): consumer rows [begin, loaded, arrive, done, s4..s7] per
// phase, in phase order, where s4..s7 are attention sub-steps (q loaded, cache pieces done,
// partial record written, combine done; 0 elsewhere); the last row of a traced CTA holds the
// producer's [cycles blocked on a free slot, cycles blocked on a KV epoch, stages issued,
// total cycles].
constexpr int kTraceWords = 8;

void launch_decode(const Params& p, void* stream, int smem_bytes, int* err);

// Read-only view of a handle's internals for entry points defined outside kd_api.cu.
struct kd_ctx_view {
    const Dims* dm;
    const Layout* lay;
    uint8_t* arena;
    void* stream;
    int device, nb, smem, ns, pieces, pos_per_stage, xs_floats, xown_floats;
    long long timeout_ns;
    int prefetch, inflight;
    bool has_weights;
};
int monokernel_smem_bytes(const Params& p);
int monokernel_occupancy(const Dims& dm, int smem_bytes, int* blocks_per_sm);

}  // namespace kd
