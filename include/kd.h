/*
 * kd.h -- C ABI of libkd: single-request (batch 1) autoregressive decode of a dense
 * decoder-only transformer on one NVIDIA B200 (sm_100a), run as ONE persistent kernel
 * per decode call.
 *
 * The problem it solves is the one the pages pose: generate the tokens of one request
 * one at a time, as fast as the memory system allows, because every generated token must
 * stream every active weight from HBM ("3000 tokens per second: how to speed up LLMs on
 * ordinary GPUs", aikraft.ru, sections 01-02; "Breaking the memory wall: 3,000 tokens/s on
 * standard GPUs", agentlenshq.com, section "The bottleneck: memory bandwidth, not
 * compute"). The decode path runs as one resident GPU program covering the matrix
 * products, attention, normalisation and sampling, with no return to the host between
 * tokens (aikraft.ru, section 04 "Monokernel and optimized GPU code"; agentlenshq.com,
 * section "1. The Monokernel Runtime").
 *
 * Model: pre-norm decoder; per layer RMSNorm -> Q/K/V projections -> RoPE (rotate-half
 * pairs (i, i+hd/2), frequency theta^(-2i/hd), absolute positions) -> bf16 KV-cache append
 * -> GQA attention (q head h reads kv head h*Hkv/Hq, scale 1/sqrt(hd)) -> output
 * projection + residual -> RMSNorm -> SwiGLU FFN (silu(gate) * up, then down) + residual;
 * then a final RMSNorm, an untied LM head and a greedy argmax (lowest index wins a tie), or,
 * after kd_set_sampling, a draw from softmax(logits / T) made inside the kernel. No biases. Weights and KV cache are bf16; all activations and accumulations are fp32.
 *
 * Memory ownership. The caller allocates every byte of device memory: one arena of
 * kd_arena_bytes() bytes (weights in the library's streaming layout, the KV cache,
 * activations and control words), the weight tensors handed to kd_load_weights, and the
 * token/logit output buffers. The library never calls cudaMalloc or cudaFree; it owns
 * only the host-side handle, freed by kd_destroy.
 *
 * Streams and threads. Every call that touches the device is asynchronous on the stream
 * given to kd_create, except kd_sync and kd_generate, which wait for it, and kd_create
 * itself, which waits once for a short probe of which B200 die owns which control word. A handle is not
 * thread-safe: use one handle per host thread and stream. kd_decode makes exactly one
 * kernel launch (a cooperative launch of one CTA per SM).
 *
 * Errors. Functions return KD_OK (0) or a negative KD_E* code. Argument, capacity and
 * co-residency errors are detected on the host before anything is launched. Errors the
 * kernel detects (a wait that exceeded its time limit, a token id outside the vocabulary)
 * are reported by kd_sync; after one, the handle refuses kd_decode until kd_reset.
 * kd_last_error() describes the last error.
 */
#ifndef KD_H
#define KD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    KD_OK = 0,
    KD_EINVAL = -1,    /* bad argument, NULL pointer or unsupported configuration */
    KD_ENOMEM = -2,    /* arena smaller than kd_arena_bytes(), or misaligned */
    KD_ECAPACITY = -3, /* position + steps would exceed max_seq */
    KD_ECOOP = -4,     /* the kernel cannot have one CTA resident on every SM */
    KD_ECUDA = -5,     /* a CUDA runtime call failed (message in kd_last_error) */
    KD_ETIMEOUT = -6,  /* a device-side wait exceeded its limit; the kernel unwound */
    KD_ESTATE = -7,    /* call out of order: no weights, nothing pending, or failed run */
    KD_ETOKEN = -8     /* a token id outside [0, vocab) reached the kernel, which stopped
                          before reading any embedding row for it */
};

/* Model shape. Limits: n_layers >= 1; head_dim in {64, 128}; n_heads a multiple of
 * n_kv_heads with n_heads / n_kv_heads <= 8; n_kv_heads <= 16; d_model a multiple of 256
 * between 256 and 8192 whose slices of at most 1024 elements are multiples of 256 (every
 * GEMV row is streamed as whole 16-byte chunks per lane: 256, 512, ..., 4096, 6144, 8192
 * qualify; 5120 does not); ffn_dim >= 1; vocab >= 1; max_seq >= 1 (KV positions held). */
typedef struct kd_config {
    int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, max_seq;
    float rms_eps, rope_theta;
} kd_config;

/* Device pointers to bf16 tensors, row-major [out][in], stacked over layers:
 *   embed [vocab][d]        attn_norm [L][d]        wq [L][Hq*hd][d]
 *   wk [L][Hkv*hd][d]       wv [L][Hkv*hd][d]       wo [L][d][Hq*hd]
 *   ffn_norm [L][d]         wg [L][F][d]            wu [L][F][d]
 *   wd [L][d][F]            final_norm [d]          lm_head [vocab][d]
 * Each must be 16-byte aligned. They are copied into the arena; the caller may free them
 * once the stream has passed kd_load_weights. */
typedef struct kd_weights {
    const void *embed, *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *wg, *wu, *wd, *final_norm,
        *lm_head;
} kd_weights;

/* Launch shape chosen by kd_create (read-only information). */
typedef struct kd_info {
    int32_t grid;          /* CTAs = SMs, one resident per SM */
    int32_t threads;       /* per CTA: 1 producer warp + consumer warps */
    int32_t smem_bytes;    /* dynamic shared memory per CTA */
    int32_t stages;        /* weight/KV pipeline stages per CTA */
    int32_t stage_bytes;   /* bytes per stage */
    int32_t attn_pieces;   /* CTAs per kv head: attention pieces, and the shares of that kv
                              head's Q/K/V rows and output-projection inputs */
    int64_t arena_bytes;   /* bytes of the arena layout */
    int64_t weight_bytes;  /* bytes of the weights inside the arena */
    int64_t kv_bytes;      /* bytes of the KV cache inside the arena */
    int64_t launches;      /* kernel launches made through this handle so far */
    int64_t ctl_offset;    /* byte offset of the control words in the arena; exposed for
                              diagnostics and tests, not to be written while a decode runs */
    int32_t sync_replicas; /* copies of the monotonic 64-bit count of cross-CTA sync arrivals:
                              2 when kd_create found the two dies of a B200 (every CTA adds to
                              both, polls the one on its own die), else 1 */
    int64_t sync_offset[2]; /* byte offsets of those copies in the arena (equal when 1) */
} kd_info;

typedef struct kd_ctx kd_ctx;

/* Bytes of device memory the arena for `cfg` needs (0 if cfg is invalid). */
size_t kd_arena_bytes(const kd_config *cfg);

/* Bytes one decode step reads by definition: every active weight once (all layers, final
 * norm, one embedding row, plus the LM head when with_head != 0) and the bf16 K and V rows
 * of kv_positions cached positions per layer and kv head. The pages' light-speed bound is
 * bandwidth divided by this (aikraft.ru, section 02). Returns -1 for an invalid cfg. */
double kd_step_bytes(const kd_config *cfg, int64_t kv_positions, int with_head);

/* Bind a handle to `d_arena` (device memory of at least kd_arena_bytes(cfg) bytes,
 * 256-byte aligned) on the current CUDA device and `stream` (a cudaStream_t, may be NULL
 * for the legacy default stream). Zeroes the control words. *out receives the handle. */
int kd_create(const kd_config *cfg, void *d_arena, size_t arena_bytes, void *stream, kd_ctx **out);

/* Copy the weights into the arena's streaming layout (a few repack kernels; not part of
 * the decode path). */
int kd_load_weights(kd_ctx *ctx, const kd_weights *w);

/* Fill positions [0, n_pos) of the K (which = 0, already rotated) or V (which = 1) cache
 * of one layer from d_src, bf16 laid out [n_kv_heads][n_pos][head_dim] in device memory. */
int kd_set_kv(kd_ctx *ctx, int32_t layer, int32_t which, const void *d_src, int32_t n_pos);

/* Start a request: positions [0, kv_len) of the cache are taken as valid (filled by
 * kd_set_kv or by earlier steps), and the n_tokens ids at d_tokens (device memory) are the
 * pending inputs, the first of them at position kv_len. Clears the error state of a failed
 * run that kd_sync reported. */
int kd_reset(kd_ctx *ctx, const int32_t *d_tokens, int32_t n_tokens, int32_t kv_len);

/* Run the pending tokens through the decoder, then generate n_gen tokens greedily, in ONE
 * kernel launch. Steps run = pending + n_gen - 1; each appends one KV position.
 * d_tokens_out: device int32 [n_gen] (may be NULL only if n_gen == 0).
 * d_logits_out: NULL, or device fp32 [steps][vocab] receiving the logits of every step,
 * prompt steps included (test use: it adds vocab*4 bytes of writes per step and makes
 * prompt steps run the LM head). Afterwards the last generated token (or, if n_gen == 0,
 * the last pending token) is pending, so calls chain. Returns KD_ECAPACITY if
 * position + steps > max_seq. */
int kd_decode(kd_ctx *ctx, int32_t n_gen, int32_t *d_tokens_out, float *d_logits_out);

/* Host-memory convenience: kd_reset with h_tokens (host int32 [n_tokens], copied to the
 * device), kd_decode(n_gen), copy the n_gen tokens to h_tokens_out (host), and wait.
 * Returns the kd_sync status. */
int kd_generate(kd_ctx *ctx, const int32_t *h_tokens, int32_t n_tokens, int32_t kv_len,
                int32_t n_gen, int32_t *h_tokens_out);

/* Time limit, in nanoseconds (>= 1), of every device-side wait of later launches: a
 * cross-CTA sync, a weight stage, a tagged activation, a KV-row guard. The default is 1 s, or
 * KD_TIMEOUT_MS milliseconds when that environment variable is set at kd_create. A wait that
 * exceeds its limit sets the device status and every CTA stops (none traps, none hangs:
 * copies already in flight are awaited under a separate fixed bound); kd_sync then returns
 * KD_ETIMEOUT and the handle needs kd_reset. Returns KD_EINVAL for ns < 1. */
int kd_set_timeout(kd_ctx *ctx, int64_t ns);

/* Token choice of later kd_decode / kd_generate / kd_decode_noalloc calls. temperature 0
 * (the default) picks the greedy argmax. temperature > 0 draws each generated token from
 * softmax(logits / temperature) inside the kernel ("3000 tokens per second", aikraft.ru,
 * section 04 "Monokernel": sampling stays on the GPU): the argmax over the vocabulary of
 * logit_i * (1/temperature) + g_i, g_i = -log(-log(u_i)) (the Gumbel-max rule, an exact draw),
 * in fp32, lowest index on a tie. u_i comes from the counter-based generator Philox4x32-10
 * (Salmon et al., SC 2011) with key (seed mod 2^32, seed div 2^32) and counter
 * (i div 4, position, 0, 0), output word i mod 4, u = (top 23 bits + 0.5) / 2^23; the position is
 * the absolute KV position of the step, so a request draws the same tokens however it is split
 * into calls. Logits written to d_logits_out stay the raw logits. Returns KD_EINVAL for a
 * negative or non-finite temperature. */
int kd_set_sampling(kd_ctx *ctx, float temperature, uint64_t seed);

/* Wait for the stream, then return the device status of the last decode (KD_OK,
 * KD_ETIMEOUT, KD_ETOKEN) or a CUDA error. */
int kd_sync(kd_ctx *ctx);

/* kd_decode without device working memory of its own: the pages have no counterpart; this
 * is a service to callers that cannot allocate device memory while decoding (for example an
 * engine whose memory pool is fully committed at start-up and forbids cudaMalloc later, or
 * a host that can only lend the library buffers it registered in advance).
 * It resets the request like kd_reset (d_tokens: device int32 [n_tokens], the first at
 * position kv_len) and generates n_gen tokens in one launch, exactly like kd_decode, but the
 * split-K sums, the tagged Q/K/V words and attention records, the control words and the
 * pending tokens live in a 1 MiB array inside the library (loaded on every GPU that loads
 * libkd, held until exit) instead of in the arena's scratch region. The weights and the KV
 * cache are still the handle's arena: the call appends to that cache at positions
 * [kv_len, kv_len + steps) like kd_decode would. Inputs and outputs as for kd_decode; returns
 * KD_EINVAL with a message when this model and n_tokens need more than the 1 MiB. It calls no
 * allocator: the scratch it uses is cleared with a memset and the tokens copied in, then it
 * waits for the launch and returns its device status. The array keeps the last call's contents and every call shares it, so
 * calls that overlap on the GPU (two streams, two handles) race: serialise them. The first
 * call on a device looks the array's address up (cudaGetSymbolAddress), so make that first
 * call outside any stream capture. The handle's position and pending tokens are not changed. */
int kd_decode_noalloc(kd_ctx *ctx, const int32_t *d_tokens, int32_t n_tokens, int32_t kv_len,
                      int32_t n_gen, int32_t *d_tokens_out, float *d_logits_out);

/* Optional phase trace for performance analysis (off by default). While set, every
 * decode launch has each CTA with index % every == 0 record, per phase (Q/K/V, attention,
 * output projection, gate/up, down, LM head) and in phase order, a row of eight words:
 * the phase id (step << 16 | layer << 4 | phase 0..5), then SM-clock stamps of phase begin,
 * inputs ready (the cross-CTA sync passed or the tagged inputs polled), compute done and
 * phase end, then the cycles spent waiting for weight / KV stages, then the stamps of the
 * phase's first and last weight / KV stage becoming ready (0 in a phase without stages).
 * Traced CTA i owns rows [i * R, (i + 1) * R) of the buffer, where
 * R = n_words / (8 * ceil(grid / every)); its last row holds the producer warp's cycles
 * blocked on a free pipeline stage, cycles blocked on KV rows written during the launch,
 * stages issued and total cycles. d_buf: device memory of n_words uint64 (caller-owned);
 * NULL turns tracing off. */
int kd_set_trace(kd_ctx *ctx, unsigned long long *d_buf, int64_t n_words, int32_t every);

/* Next KV position to be written (host-side view, valid once calls were enqueued). */
int32_t kd_position(const kd_ctx *ctx);

int kd_get_info(const kd_ctx *ctx, kd_info *info);

/* Device address of one layer's K (which = 0) or V (which = 1) cache, laid out
 * [n_kv_heads][max_seq][head_dim] bf16; NULL on a bad argument. */
void *kd_kv_ptr(kd_ctx *ctx, int32_t layer, int32_t which);

const char *kd_last_error(const kd_ctx *ctx);
const char *kd_strerror(int code);

/* Free the host handle (the caller still owns the arena). */
void kd_destroy(kd_ctx *ctx);

#ifdef __cplusplus
}
#endif
#endif /* KD_H */
