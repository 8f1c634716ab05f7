// kd_layout.h -- arena layout, launch constants and kernel parameters shared by the host
// side of libkd (kd_api.cu, kd_noalloc.cu) and the monokernel (kd_kernel.cu). Internal to libkd.
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define KD_HD __host__ __device__
#else
#define KD_HD
#endif

namespace kd {

// One CTA per SM: one producer warp streams weight / KV tiles into a ring of shared-memory
// stages with 1-D bulk copies; 16 consumer warps share every stage.
constexpr int kStageBytes = 32768;
constexpr int kConsumerWarps = 16;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kMaxStages = 8;
constexpr int kMaxGroup = 8;        // q heads per kv head
constexpr int kMaxKvHeads = 16;
constexpr int kMaxModel = 8192;     // d_model
constexpr int kSmemLimit = 232448;  // opt-in dynamic shared memory per CTA on B200

// Control words (uint64), each on its own 128-byte line.
constexpr int kCtlSync = 0;     // the sync counter of kd_decode_noalloc (kd_decode uses Params.sync_off)
constexpr int kCtlStatus = 16;  // 0 = ok, else an error code (device side)
constexpr int kCtlWhere = 17;   // where a wait gave up (diagnosis)
constexpr int kCtlArgmax = 32;  // 3 rotating argmax slots at kCtlArgmax + 16*i
constexpr int kCtlWords = 80;

// Die-local sync counters. A B200 spreads its SMs and its L2 over two dies; an atomic on a
// line homed on the far die takes about twice the round trip of one on the near die. kd_create
// probes kDieCandidates words kDieBlock bytes apart (the die owning a line changes at that
// granularity or coarser), keeps the first candidate and the first one homed on the other die
// as the two replicas of the sync counter, and records per SM id which replica is local.
constexpr int kDieCandidates = 16;
constexpr int kDieBlock = 2048;
constexpr int kMaxSmid = 256;

// Each cross-CTA sum is kept in kSumCopies copies: CTA c adds its partial vector into copy
// c % kSumCopies and a reader adds the copies. Half the atomics land on each copy's lines (a
// standalone round of 148 CTAs adding 8 KB and reading the sum back: 2.34 us with one copy,
// 1.99 us with two, 2.42 us with four).
constexpr int kSumCopies = 2;

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
    // within a layer block: the two norm gains, then the matrices in streaming order:
    //   wqkv [Hkv][(r + 2) * hd][d]  per kv head: its r q heads, its k head, its v head; q and k
    //                                rows in RoPE-pair order (row 2i = dim i, 2i + 1 = dim i + hd/2)
    //   wot  [Hq * hd][d]            the output projection transposed (row = attention dim)
    //   wgu  [2F][d]                 gate and up rows interleaved (2j = gate j, 2j + 1 = up j)
    //   wdt  [F][d]                  the down projection transposed (row = hidden unit)
    size_t l_attn_norm, l_ffn_norm, l_wqkv, l_wot, l_wgu, l_wdt;
    size_t rope;            // [S][hd/2] float2 (cos, sin)
    size_t kcache, vcache;  // [L][Hkv][S][hd] bf16
    // Scratch written during a launch:
    //   delta [3][kSumCopies][d] fp32 -- cross-CTA sums of the split-K output and down
    //                          projections, in kSumCopies partial copies each
    //   qkv [Hkv][(r + 2) * hd] tagged words -- RoPE'd q, RoPE'd bf16 k, bf16 v of the step
    //   rec [grid][r][hd + 2] tagged words   -- attention piece records (max, sum, acc[hd])
    size_t delta, qkv, rec;
    size_t ctl;
    size_t syncw;   // the die probe candidates / sync counter replicas (kDieBlock-aligned inside)
    size_t dietab;  // [kMaxSmid] uint8: the replica local to each SM id (written at kd_create)
    size_t tokens_in, tokens_out;
    size_t weights_end, kv_bytes, total;
};

// Shapes of the two GEMV kinds for a model of width d (both stream rows of d bf16 elements):
//  row GEMV (Q/K/V, gate/up, LM head): a row is cut into gs slices of at most 1024 elements
//    (512 up to d = 2048 where d splits so), a stage holds gr rows, and the 16 consumer warps
//    share the gr * gs (row, slice) units of a stage, gm = gr * gs / 16 each;
//  split-K GEMV (output and down projections): a stage holds kr rows; thread t owns the
//    8 outputs of chunk t % (d / 8) and the rows t / (d / 8) + k * ug of each stage.
struct Shape {
    int gs, gr, gm;  // row GEMV
    int kr, ug, kc;  // split-K GEMV: rows per stage, unit groups, output chunks per thread
};
inline bool make_shape(int d, Shape* s) {
    if (d < 256 || d % 256 || d > kMaxModel) return false;
    // Slices of at most 1024 elements; up to d = 2048, of at most 512 where d splits so (each
    // warp then holds 16 activation values per lane and reads half as much of the activation
    // vector per phase: 2.7% per token on the 2B model; neutral on the 8B model, which keeps
    // 1024).
    const int smax = d <= 2048 ? 512 : 1024;
    int gs = 1;
    while (d / gs > smax && (d / (2 * gs)) % 256 == 0) gs *= 2;
    if (d / gs > 1024 || (d / gs) % 256) return false;
    const int maxr = kStageBytes / (2 * d);
    const int unit = kConsumerWarps / gs;  // rows must come in multiples of this
    int gr = (maxr / unit) * unit;
    if (gr > 64) gr = 64;
    if (gr < unit) return false;
    s->gs = gs;
    s->gr = gr;
    s->gm = gr * gs / kConsumerWarps;
    if (s->gm != 1 && s->gm != 2 && s->gm != 4) return false;
    const int oc = d / 8;
    s->kr = maxr > 64 ? 64 : maxr;
    s->ug = oc >= kConsumerThreads ? 1 : kConsumerThreads / oc;
    s->kc = (oc + kConsumerThreads - 1) / kConsumerThreads;
    if (s->kc > 2) return false;
    return true;
}

// Bytes reserved for the sync counter replicas (alignment slack included).
KD_HD inline size_t sync_region_bytes() { return (size_t)(kDieCandidates + 1) * kDieBlock; }

// Cross-CTA sums ("syncs") per decode step: the output projection and the down projection of
// every layer, then the argmax of the steps that run the LM head (all steps when logits are
// dumped). Sync k adds into delta buffer k % 3 (its kSumCopies copies).
KD_HD inline long long syncs_before_step(int L, int s, int n_pending, bool dump) {
    const long long heads = dump ? s : (s - (n_pending - 1) > 0 ? s - (n_pending - 1) : 0);
    return 2LL * L * s + heads;
}
// Tagged phases (Q/K/V outputs and attention records) a launch of `steps` steps writes: two per
// layer and step. Tags of successive launches follow each other, so a word never carries a
// stale tag that a reader of a later launch expects.
KD_HD inline long long launch_tags(int L, int steps) { return 2LL * L * steps; }

struct Params {
    // weights (arena)
    const uint8_t* arena;
    Layout lay;
    Dims dm;
    Shape sh;
    // per-launch
    int steps;      // decode steps in this launch
    int n_pending;  // tokens fed before the first generated one
    int pos0;       // position of step 0
    int n_gen;
    int dump;       // write logits of every step
    int32_t* tokens_out;
    float* logits_out;
    // token choice: greedy when inv_temp == 0, else the Gumbel-max draw with this seed
    float inv_temp;
    uint32_t seed_lo, seed_hi;
    // sync counter: nsync replicas (1 or 2) at these arena byte offsets; every CTA adds to all
    // of them and polls the one local to its SM (lay.dietab)
    size_t sync_off[2];
    int nsync;
    // launch shape
    int nb;         // CTAs
    int ns;         // pipeline stages
    int pieces;     // CTAs per kv head (attention pieces, and the Q/K/V and output-projection shares)
    int blk;        // positions per attention softmax block
    int work_floats, hin_floats;  // shared-memory scratch sizes
    long long timeout_ns;
    uint32_t tag0;  // tagged phase i of this launch tags its words tag0 + 1 + i
    // optional trace: CTAs with blockIdx.x % trace_every == 0 record per-phase timestamps
    unsigned long long* trace;
    int trace_every, trace_rows;
};

// Trace row layout (SM clock cycles), one row per phase of a traced CTA, in phase order:
// [phase id (step << 16 | layer << 4 | phase), begin, inputs ready, compute done, end,
//  cycles waiting for weight / KV stages, first stage ready, last stage ready] (the last two
//  are 0 in a phase without stages). The last row of a traced CTA holds the
// producer warp's [cycles waiting for a free stage, cycles waiting for KV rows written this
// launch, stages issued, total cycles].
constexpr int kTraceWords = 8;

void launch_decode(const Params& p, void* stream, int smem_bytes, int* err);

// Read-only view of a handle's internals for entry points defined outside kd_api.cu.
struct kd_ctx_view {
    const Dims* dm;
    const Layout* lay;
    const Shape* sh;
    uint8_t* arena;
    void* stream;
    int device, nb, smem, ns, pieces, blk, work_floats, hin_floats;
    long long timeout_ns;
    bool has_weights;
    float inv_temp;
    unsigned long long seed;
    size_t sync_off[2];
    int nsync;
};
int monokernel_smem_bytes(const Params& p);
int monokernel_occupancy(const Dims& dm, int smem_bytes, int* blocks_per_sm);

}  // namespace kd
