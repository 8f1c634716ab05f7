// kd_noalloc.cu -- kd_decode_noalloc: the decode launch with its working memory taken from
// a fixed array that the library itself carries, so the call needs no device allocation.
//
// Who needs this: callers that cannot allocate device memory at decode time. Examples are
// an engine whose memory pool is fully committed to weights and caches and which forbids
// cudaMalloc after start-up, a host that only hands the library pre-registered buffers, and
// code paths where an allocation could fail or stall mid-request. Such a caller still owns
// the weights and the KV cache (the handle's arena from kd_create) and its own input and
// output buffers; the split-K sums, the exchange words (Q/K/V outputs and attention records),
// the control words and the pending-token list live here instead of in the arena's scratch
// region.
#include <cuda_runtime.h>
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "kd.h"
#include "kd_layout.h"

using namespace kd;

int kd_internal_view(kd_ctx* ctx, kd_ctx_view* v);
namespace kd {
void fill_launch_shape(const kd_ctx_view& v, Params& p);
}
int kd_internal_fail(kd_ctx* ctx, int code, const char* msg);
void kd_internal_count_launch(kd_ctx* ctx);

// The scratch array: loaded onto every GPU that loads libkd and held there until the
// process exits. Its size caps what one call can use (see kd_decode_noalloc in kd.h).
constexpr size_t kNoallocScratchBytes = 1u << 20;
static __device__ __align__(256) unsigned char kd_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices];  // device address of kd_noalloc_scratch per device, once resolved

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Resolve the array's device address on the current device (first call per device only).
cudaError_t scratch_address(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, kd_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return cudaSuccess;
}

}  // namespace


extern "C" int kd_decode_noalloc(kd_ctx* ctx, const int32_t* d_tokens, int32_t n_tokens, int32_t kv_len,
                                 int32_t n_gen, int32_t* d_tokens_out, float* d_logits_out) {
    kd_ctx_view v;
    if (!ctx || kd_internal_view(ctx, &v) != KD_OK) return KD_EINVAL;
    if (!v.has_weights) return kd_internal_fail(ctx, KD_ESTATE, "kd_decode_noalloc: no weights loaded");
    if (!d_tokens || n_tokens < 1 || n_gen < 0 || (n_gen > 0 && !d_tokens_out) || kv_len < 0)
        return kd_internal_fail(ctx, KD_EINVAL, "kd_decode_noalloc: bad tokens, n_gen or kv_len");
    const Dims& dm = *v.dm;
    const int steps = n_tokens + n_gen - 1;
    if ((long long)kv_len + steps > dm.S)
        return kd_internal_fail(ctx, KD_ECAPACITY, "kd_decode_noalloc: kv_len + steps exceeds max_seq");

    // this call's slice of the array: the same regions the arena reserves for scratch
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = up256(off + bytes);
        return at;
    };
    const size_t o_delta = take((size_t)3 * kSumCopies * dm.d * 4);
    const size_t o_qkv = take((size_t)dm.qkv_rows * 8);
    const size_t o_rec = take((size_t)v.nb * dm.r * (dm.hd + 2) * 8);
    const size_t o_ctl = take((size_t)kCtlWords * 8);
    const size_t o_tok = take((size_t)n_tokens * 4);
    if (off > kNoallocScratchBytes) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "kd_decode_noalloc: needs %zu bytes of scratch for this model and %d tokens, above the %zu-byte "
                 "maximum",
                 off, n_tokens, kNoallocScratchBytes);
        return kd_internal_fail(ctx, KD_EINVAL, msg);
    }
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess || cur != v.device || cur < 0 || cur >= kMaxDevices)
        return kd_internal_fail(ctx, KD_EINVAL, "kd_decode_noalloc: make the handle's device current");
    void* base = nullptr;
    if ((e = scratch_address(cur, &base)) != cudaSuccess)
        return kd_internal_fail(ctx, KD_ECUDA, cudaGetErrorString(e));
    uint8_t* s = static_cast<uint8_t*>(base);

    // The split-K buffers, tagged words and control words must start at zero (the array keeps
    // the previous call's contents, possibly another handle's, so tags restart at 1 each
    // call); the pending tokens are copied in. None of this allocates.
    if ((e = cudaMemsetAsync(s + o_delta, 0, o_tok - o_delta, (cudaStream_t)v.stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(s + o_tok, d_tokens, (size_t)n_tokens * 4, cudaMemcpyDeviceToDevice, (cudaStream_t)v.stream)) !=
            cudaSuccess)
        return kd_internal_fail(ctx, KD_ECUDA, cudaGetErrorString(e));
    if (steps == 0) return KD_OK;

    // The kernel addresses every region as arena + offset; scratch offsets are taken
    // relative to the arena so that they land in the array (64-bit wrap-around addition).
    auto rel = [&](size_t o) { return (size_t)((uintptr_t)(s + o) - (uintptr_t)v.arena); };
    Params p{};
    fill_launch_shape(v, p);
    p.arena = v.arena;
    p.lay = *v.lay;
    p.lay.delta = rel(o_delta), p.lay.qkv = rel(o_qkv), p.lay.rec = rel(o_rec);
    p.lay.ctl = rel(o_ctl), p.lay.tokens_in = rel(o_tok);
    // one sync counter, in this call's control words (the handle's die-local replicas stay
    // the handle's)
    p.sync_off[0] = p.sync_off[1] = rel(o_ctl) + (size_t)kCtlSync * 8;
    p.nsync = 1;
    p.steps = steps;
    p.n_pending = n_tokens;
    p.pos0 = kv_len;
    p.n_gen = n_gen;
    p.dump = d_logits_out != nullptr;
    p.tokens_out = d_tokens_out;
    p.logits_out = d_logits_out;
    p.tag0 = 0;
    int err = 0;
    launch_decode(p, v.stream, v.smem, &err);
    if (err != 0) return kd_internal_fail(ctx, KD_ECUDA, cudaGetErrorString((cudaError_t)err));
    kd_internal_count_launch(ctx);
    // The status word of this launch is in the array, so the call waits for the launch and
    // reads it back itself (into host memory; nothing is allocated).
    unsigned long long status = 0;
    if ((e = cudaMemcpyAsync(&status, s + o_ctl + (size_t)kCtlStatus * 8, sizeof status, cudaMemcpyDeviceToHost,
                             (cudaStream_t)v.stream)) != cudaSuccess ||
        (e = cudaStreamSynchronize((cudaStream_t)v.stream)) != cudaSuccess)
        return kd_internal_fail(ctx, KD_ECUDA, cudaGetErrorString(e));
    if (status == (unsigned long long)kStatusToken)
        return kd_internal_fail(ctx, KD_ETOKEN, "kd_decode_noalloc: a token id outside [0, vocab) reached the kernel");
    if (status != 0) return kd_internal_fail(ctx, KD_ETIMEOUT, "kd_decode_noalloc: a device-side wait exceeded its limit");
    return KD_OK;
}
