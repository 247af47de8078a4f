// api.cu -- C ABI entry points (include/rfx.h): argument checks, workspace
// layout and kernel launches.  No entry point allocates device memory except
// moe_layer_create_mix (its per-expert table, made once per layer).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/rfx.h"
#include "gemv.h"
#include "moe_decode.h"
#include "prefill.h"
#include "rfx_layout.h"
#include "stack.h"

int rfx_fail(int code, const std::string& msg);  // rfx_pack.cpp

struct moe_layer {
    moe_layer_desc d;
    rfx::MoeMixEntry* mix_dev = nullptr;   // ROCmFPX MIX: device table [E], else null
    int mix_count[5] = {0, 0, 0, 0, 0};    // routed experts per gate/up format (MIX)
    // moe_ffn_forward_host: the uploads run on a stream of their own into two
    // buffer sets used in turn, so that a call's uploads overlap the previous
    // call's kernels (made on first use; calls on one layer are serialised)
    std::mutex host_mu;
    cudaStream_t up_stream = nullptr;
    cudaEvent_t ev_free[2] = {nullptr, nullptr}, ev_ready[2] = {nullptr, nullptr};
    unsigned host_calls = 0;
};

namespace {

bool fmt_ok(int f) { return f == 2 || f == 3 || f == 4; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int cuda_fail(const char* where, cudaError_t e) {
    return rfx_fail(RFX_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

// SM count and opt-in shared memory of the current device, queried once per
// device (thread-safe: the shared-memory size is published before the SM
// count, and a reader that sees the count sees the size).
int device_props(int& sms, int& smem_optin) {
    static std::atomic<int> cache_sms[64] = {}, cache_smem[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    const bool cached = dev >= 0 && dev < 64;
    if (cached) {
        const int s = cache_sms[dev].load(std::memory_order_acquire);
        if (s) {
            sms = s;
            smem_optin = cache_smem[dev].load(std::memory_order_relaxed);
            return RFX_OK;
        }
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
    e = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
    if (cached) {
        cache_smem[dev].store(smem_optin, std::memory_order_relaxed);
        cache_sms[dev].store(sms, std::memory_order_release);
    }
    return RFX_OK;
}

}  // namespace

extern "C" int rfx_pack_device(rfx_format f, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols,
                               void* dst, void* stream) {
    if (!fmt_ok(f)) return rfx_fail(RFX_EINVAL, "rfx_pack_device: bad format");
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return rfx_fail(RFX_EINVAL, "rfx_pack_device: bad shape");
    if (rows > 65535LL * 16) return rfx_fail(RFX_EUNSUPPORTED, "rfx_pack_device: more than 1048560 rows");
    if (rows == 0) return RFX_OK;
    if (!codes || !scales || !dst) return rfx_fail(RFX_EINVAL, "rfx_pack_device: null pointer");
    cudaError_t e = rfx::pack_device_launch(f, codes, scales, rows, cols, (uint8_t*)dst, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("rfx_pack_device", e);
}

extern "C" int moe_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, void* stream) {
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 16)
        return rfx_fail(RFX_EINVAL, "moe_router_topk: need T >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 16)");
    if (T == 0) return RFX_OK;
    if (!logits || !idx || !w) return rfx_fail(RFX_EINVAL, "moe_router_topk: null pointer");
    cudaError_t e = rfx::router_topk_launch(logits, T, E, k, idx, w, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("moe_router_topk", e);
}

extern "C" int moe_router_logits(const void* w_router, const float* bias, const void* x, int T, int H, int E,
                                 float* logits, void* stream) {
    if (T < 0 || E < 1 || H < 32 || H % 32 != 0)
        return rfx_fail(RFX_EINVAL, "moe_router_logits: need T >= 0, E >= 1 and H a positive multiple of 32");
    if ((long long)T > 8LL * 65535) return rfx_fail(RFX_EUNSUPPORTED, "moe_router_logits: T <= 524280");
    if (T == 0) return RFX_OK;
    if (!w_router || !x || !logits) return rfx_fail(RFX_EINVAL, "moe_router_logits: null pointer");
    if (((uintptr_t)w_router & 15u) || ((uintptr_t)x & 15u))
        return rfx_fail(RFX_EINVAL, "moe_router_logits: w_router and x must be 16-byte aligned");
    cudaError_t e = rfx::router_logits_launch((const uint16_t*)w_router, bias, (const uint16_t*)x, T, H, E, logits,
                                              (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("moe_router_logits", e);
}

extern "C" int moe_router_project_topk(const void* w_router, const float* bias, const void* x, int T, int H, int E,
                                       int k, float* logits, int32_t* idx, float* w, void* stream) {
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 16)
        return rfx_fail(RFX_EINVAL, "moe_router_project_topk: need T >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 16)");
    if (T >= 1 && T <= 8) {   // decode / verify: projection and top-k in one cooperative launch
        if (H < 32 || H % 32 != 0) return rfx_fail(RFX_EINVAL, "moe_router_project_topk: H a positive multiple of 32");
        if (!w_router || !x || !logits || !idx || !w) return rfx_fail(RFX_EINVAL, "moe_router_project_topk: null pointer");
        if (((uintptr_t)w_router & 15u) || ((uintptr_t)x & 15u))
            return rfx_fail(RFX_EINVAL, "moe_router_project_topk: w_router and x must be 16-byte aligned");
        cudaError_t e = rfx::router_project_topk_launch((const uint16_t*)w_router, bias, (const uint16_t*)x, T, H, E, k,
                                                        logits, idx, w, (cudaStream_t)stream);
        if (e != cudaErrorNotSupported) return e == cudaSuccess ? RFX_OK : cuda_fail("moe_router_project_topk", e);
        // the grid does not fit the device at once: the two launches below
    }
    int rc = moe_router_logits(w_router, bias, x, T, H, E, logits, stream);
    if (rc != RFX_OK) return rc;
    return moe_router_topk(logits, T, E, k, idx, w, stream);
}

extern "C" int rfx_gemv_q(rfx_format f, const void* W, int64_t N, int64_t K, const void* x, int x_is_fp32, int q,
                          float* y, void* stream) {
    if (!fmt_ok(f)) return rfx_fail(RFX_EINVAL, "rfx_gemv_q: bad format");
    if (N < 1 || K < 32 || K % 32 != 0) return rfx_fail(RFX_EINVAL, "rfx_gemv_q: need N >= 1 and K a positive multiple of 32");
    if (q < 1 || q > 8) return rfx_fail(RFX_EUNSUPPORTED, "rfx_gemv_q: 1 <= q <= 8");
    if (!W || !x || !y) return rfx_fail(RFX_EINVAL, "rfx_gemv_q: null pointer");
    if (!aligned16(W)) return rfx_fail(RFX_EINVAL, "rfx_gemv_q: W must be 16-byte aligned");
    if (((uintptr_t)x & 3u) != 0) return rfx_fail(RFX_EINVAL, "rfx_gemv_q: x must be 4-byte aligned");
    int sms = 0, smem_optin = 0;
    int rc = device_props(sms, smem_optin);
    if (rc != RFX_OK) return rc;
    if (rfx::gemv_smem_bytes(q, K, x_is_fp32 != 0) > (size_t)smem_optin)
        return rfx_fail(RFX_EUNSUPPORTED, "rfx_gemv_q: q*K too large for the shared-memory copy of x");
    if ((N + 15) / 16 > 2LL * 2147483647LL) return rfx_fail(RFX_EUNSUPPORTED, "rfx_gemv_q: N too large");
    rfx::GemvParams p{(const uint8_t*)W, N, K, x, q, y};
    cudaError_t e = rfx::gemv_launch(p, f, x_is_fp32 != 0, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("rfx_gemv_q", e);
}

extern "C" int moe_layer_create(const moe_layer_desc* d, moe_layer** out) {
    if (!d || !out) return rfx_fail(RFX_EINVAL, "moe_layer_create: null pointer");
    *out = nullptr;
    if (d->H < 32 || d->I < 32 || d->H % 32 || d->I % 32)
        return rfx_fail(RFX_EINVAL, "moe_layer_create: H and I must be positive multiples of 32");
    if (d->E < 1 || d->E > 1024 || d->k < 1 || d->k > d->E || d->k > MOE_MAXK)
        return rfx_fail(RFX_EINVAL, "moe_layer_create: need 1 <= k <= min(E, 8), E <= 1024");
    if (!fmt_ok(d->f_gate) || !fmt_ok(d->f_up) || !fmt_ok(d->f_down))
        return rfx_fail(RFX_EINVAL, "moe_layer_create: bad routed format");
    if (d->f_gate != d->f_up) return rfx_fail(RFX_EUNSUPPORTED, "moe_layer_create: gate and up must share a format");
    if (!d->gate || !d->up || !d->down) return rfx_fail(RFX_EINVAL, "moe_layer_create: null routed pointer");
    if (!aligned16(d->gate) || !aligned16(d->up) || !aligned16(d->down) || d->stride_gate % 16 ||
        d->stride_up % 16 || d->stride_down % 16)
        return rfx_fail(RFX_EINVAL, "moe_layer_create: routed bases and strides must be 16-byte aligned");
    if (d->stride_gate < rfx_packed_bytes(d->f_gate, d->I, d->H) || d->stride_up < rfx_packed_bytes(d->f_up, d->I, d->H) ||
        d->stride_down < rfx_packed_bytes(d->f_down, d->H, d->I))
        return rfx_fail(RFX_EINVAL, "moe_layer_create: expert stride smaller than the packed matrix");
    if (d->has_shared) {
        if (!fmt_ok(d->f_sh_gate) || !fmt_ok(d->f_sh_up) || !fmt_ok(d->f_sh_down))
            return rfx_fail(RFX_EINVAL, "moe_layer_create: bad shared format");
        if (d->f_sh_gate != d->f_sh_up)
            return rfx_fail(RFX_EUNSUPPORTED, "moe_layer_create: shared gate and up must share a format");
        if (!d->sh_gate || !d->sh_up || !d->sh_down) return rfx_fail(RFX_EINVAL, "moe_layer_create: null shared pointer");
        if (!aligned16(d->sh_gate) || !aligned16(d->sh_up) || !aligned16(d->sh_down))
            return rfx_fail(RFX_EINVAL, "moe_layer_create: shared pointers must be 16-byte aligned");
    }
    moe_layer* L = new (std::nothrow) moe_layer;
    if (!L) return rfx_fail(RFX_EINVAL, "moe_layer_create: out of host memory");
    L->d = *d;
    *out = L;
    return RFX_OK;
}

extern "C" int moe_layer_create_mix(const moe_layer_desc* d, const moe_expert_mix* mix, moe_layer** out) {
    if (!d || !mix || !out) return rfx_fail(RFX_EINVAL, "moe_layer_create_mix: null pointer");
    *out = nullptr;
    // the descriptor's own checks, with routed formats and strides that always pass
    moe_layer_desc u = *d;
    u.f_gate = u.f_up = u.f_down = RFX_FP4;
    u.stride_gate = u.stride_up = (rfx_packed_bytes(RFX_FP4, d->I, d->H) + 15) / 16 * 16;   // FP4 packs largest
    u.stride_down = (rfx_packed_bytes(RFX_FP4, d->H, d->I) + 15) / 16 * 16;
    moe_layer* L = nullptr;
    int rc = moe_layer_create(&u, &L);
    if (rc != RFX_OK) return rc;
    std::vector<rfx::MoeMixEntry> tab((size_t)d->E);
    for (int e = 0; e < d->E; ++e) {
        const moe_expert_mix& m = mix[e];
        if (!fmt_ok(m.f_gate_up) || !fmt_ok(m.f_down)) {
            moe_layer_destroy(L);
            return rfx_fail(RFX_EINVAL, "moe_layer_create_mix: bad format in entry " + std::to_string(e));
        }
        if (m.off_gate % 16 || m.off_up % 16 || m.off_down % 16) {
            moe_layer_destroy(L);
            return rfx_fail(RFX_EINVAL, "moe_layer_create_mix: offsets must be multiples of 16 (entry " +
                                            std::to_string(e) + ")");
        }
        tab[e] = rfx::MoeMixEntry{(long long)m.off_gate, (long long)m.off_up, (long long)m.off_down, (int)m.f_gate_up,
                                  (int)m.f_down};
        ++L->mix_count[m.f_gate_up];
    }
    // the routed formats the descriptor reports: the most common ones
    int fa = 2, fb = 2, cb[5] = {0, 0, 0, 0, 0};
    for (int f = 2; f <= 4; ++f)
        if (L->mix_count[f] > L->mix_count[fa]) fa = f;
    for (int e = 0; e < d->E; ++e) ++cb[mix[e].f_down];
    for (int f = 2; f <= 4; ++f)
        if (cb[f] > cb[fb]) fb = f;
    L->d = *d;
    L->d.f_gate = L->d.f_up = (rfx_format)fa;
    L->d.f_down = (rfx_format)fb;
    L->d.stride_gate = L->d.stride_up = L->d.stride_down = 0;
    cudaError_t e = cudaMalloc(&L->mix_dev, tab.size() * sizeof(rfx::MoeMixEntry));
    if (e == cudaSuccess) e = cudaMemcpy(L->mix_dev, tab.data(), tab.size() * sizeof(rfx::MoeMixEntry), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        moe_layer_destroy(L);
        return cuda_fail("moe_layer_create_mix", e);
    }
    *out = L;
    return RFX_OK;
}

extern "C" void moe_layer_destroy(moe_layer* layer) {
    if (!layer) return;
    if (layer->mix_dev) cudaFree(layer->mix_dev);
    for (int i = 0; i < 2; ++i) {
        if (layer->ev_free[i]) cudaEventDestroy(layer->ev_free[i]);
        if (layer->ev_ready[i]) cudaEventDestroy(layer->ev_ready[i]);
    }
    if (layer->up_stream) cudaStreamDestroy(layer->up_stream);
    delete layer;
}

extern "C" size_t moe_prefill_workspace_bytes(const moe_layer* layer, int T);

extern "C" size_t moe_ffn_workspace_bytes(const moe_layer* layer, int T) {
    if (!layer || T < 1) return 0;
    if (T > MOE_MAXT) return moe_prefill_workspace_bytes(layer, T);
    return rfx::moe_ws_layout(T, layer->d.k, layer->d.H, layer->d.I).total;
}

// Bytes at the start of a workspace that hold control words (they must be
// zero before a call; the kernels return them to zero when they finish): the
// decode control block for T <= 8, the prefill one above.
size_t rfx_moe_ctrl_bytes(const moe_layer* layer, int T) {
    if (!layer) return 0;
    if (T > MOE_MAXT) return rfx::pf_ws_layout(T, layer->d.k, layer->d.E, layer->d.H, layer->d.I).cnt;
    return (size_t)MOE_CTRL_WORDS * 4;
}

// Test hook for the device error path (rfx.h): a fault to inject and a wait
// limit for later moe_ffn_forward / moe_ffn_prefill launches.
namespace {
std::atomic<int> g_fault{0};
std::atomic<long long> g_wait{0};
}  // namespace

extern "C" int rfx_debug_set_fault(int fault, long long wait_cycles) {
    if (fault < 0 || fault > 3 || wait_cycles < 0) return rfx_fail(RFX_EINVAL, "rfx_debug_set_fault: bad argument");
    g_fault.store(fault);
    g_wait.store(wait_cycles);
    return RFX_OK;
}

namespace rfx {
long long moe_default_wait_limit();
int debug_fault() { return g_fault.load(); }
long long debug_wait(long long dflt) {
    const long long w = g_wait.load();
    return w > 0 ? w : dflt;
}
}  // namespace rfx

extern "C" int rfx_ws_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws) return rfx_fail(RFX_EINVAL, "rfx_ws_init: null workspace");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("rfx_ws_init", e);
}

extern "C" int rfx_ws_status(void* ws, void* stream) {
    if (!ws) return rfx_fail(RFX_EINVAL, "rfx_ws_status: null workspace");
    uint32_t err = 0;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail("rfx_ws_status", e);
    e = cudaMemcpy(&err, (uint32_t*)ws + MOE_CTRL_ERR, 4, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail("rfx_ws_status", e);
    if (err) {
        uint32_t zero = 0;
        e = cudaMemcpy((uint32_t*)ws + MOE_CTRL_ERR, &zero, 4, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail("rfx_ws_status", e);
    }
    if (err & MOE_ERR_TIMEOUT) return rfx_fail(RFX_EDEVICE, "device: a bounded wait timed out");
    if (err & MOE_ERR_EXPERT) return rfx_fail(RFX_EDEVICE, "device: expert id out of range");
    if (err & MOE_ERR_RANGE) return rfx_fail(RFX_ERANGE, "device: a SwiGLU intermediate is not a finite fp32 value");
    return RFX_OK;
}

namespace rfx {

// Fill launch parameters for T columns; returns RFX_OK or an error.
// The staged x copies of the decode kernel (one per gate/up format that gets
// its own, at most two): the most common routed format first, then the shared
// expert's, else the next most common routed one.  A slot of any other format
// reads copy 0 and corrects its scales.
void x_copies(const moe_layer* layer, int& nxc, int xf[2], int& other) {
    const moe_layer_desc& d = layer->d;
    int cnt[5] = {0, 0, 0, 0, 0};
    if (layer->mix_dev)
        for (int f = 2; f <= 4; ++f) cnt[f] = layer->mix_count[f];
    else
        cnt[d.f_gate] = d.E;
    int f0 = d.f_gate;
    for (int f = 2; f <= 4; ++f)
        if (cnt[f] > cnt[f0]) f0 = f;
    xf[0] = f0;
    xf[1] = f0;
    nxc = 1;
    if (d.has_shared && d.f_sh_gate != f0) {
        xf[1] = d.f_sh_gate;
        nxc = 2;
    } else {
        int f1 = 0;
        for (int f = 2; f <= 4; ++f)
            if (f != f0 && cnt[f] > 0 && (f1 == 0 || cnt[f] > cnt[f1])) f1 = f;
        if (f1) {
            xf[1] = f1;
            nxc = 2;
        }
    }
    other = 0;
    for (int f = 2; f <= 4; ++f)
        if (cnt[f] > 0 && f != xf[0] && f != xf[1]) other = 1;
}

int moe_prepare(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w, float* y, void* ws,
                size_t ws_bytes, MoeParams& p, int& grid, size_t& smem) {
    if (!layer) return rfx_fail(RFX_EINVAL, "moe_ffn_forward: null layer");
    const moe_layer_desc& d = layer->d;
    if (T < 1 || T > MOE_MAXT) return rfx_fail(RFX_EUNSUPPORTED, "moe_ffn_forward: 1 <= T <= 8 token columns");
    if (!x || !idx || !w || !y || !ws) return rfx_fail(RFX_EINVAL, "moe_ffn_forward: null pointer");
    if (((uintptr_t)x & 15u) || ((uintptr_t)ws & 255u))
        return rfx_fail(RFX_EINVAL, "moe_ffn_forward: x must be 16-byte and ws 256-byte aligned");
    const MoeWs L = moe_ws_layout(T, d.k, d.H, d.I);
    if (ws_bytes < L.total) return rfx_fail(RFX_EINVAL, "moe_ffn_forward: workspace smaller than moe_ffn_workspace_bytes");
    int sms = 0, smem_optin = 0;
    int rc = device_props(sms, smem_optin);
    if (rc != RFX_OK) return rc;
    p.H = d.H; p.I = d.I; p.E = d.E; p.k = d.k; p.T = T;
    p.fA = d.f_gate; p.fB = d.f_down;
    p.fsA = d.has_shared ? d.f_sh_gate : 2;
    p.fsB = d.has_shared ? d.f_sh_down : 2;
    p.gate = (const uint8_t*)d.gate; p.up = (const uint8_t*)d.up; p.down = (const uint8_t*)d.down;
    p.sg = (long long)d.stride_gate; p.su = (long long)d.stride_up; p.sd = (long long)d.stride_down;
    p.mix = layer->mix_dev;
    x_copies(layer, p.nxc, p.xf, p.other);
    p.has_shared = d.has_shared ? 1 : 0;
    p.shg = (const uint8_t*)d.sh_gate; p.shu = (const uint8_t*)d.sh_up; p.shd = (const uint8_t*)d.sh_down;
    p.x = (const uint16_t*)x; p.xc = nullptr; p.idx = idx; p.wts = w; p.y = y;
    uint8_t* wsb = (uint8_t*)ws;
    p.ctrl = (uint32_t*)(wsb + L.ctrl_off);
    p.hfrag = wsb + L.hf_off;
    p.dpart = (float*)(wsb + L.d_off);
    p.hslot_bytes = (long long)L.hslot;
    p.wait_limit = debug_wait(moe_default_wait_limit());
    p.fault = debug_fault();
    if (p.fault > 2) p.fault = 0;
    p.x_stride = d.H / 16 * 32 + 32;
    // Shared memory: the ring, the staged x (gate/up phase: one copy per
    // gate/up format in use, and its block sums) and two h buffers (down
    // phase), the reduction buffers.  An h buffer placed over the staged x is
    // filled only once this CTA's gate/up stages are consumed, so the plans
    // that keep the first (or both) buffers clear of x come first.
    const int qc = moe_qclass(T);
    auto r128 = [](size_t n) { return (n + 127) / 128 * 128; };
    const int nxc = p.nxc;
    const size_t xb = r128((size_t)nxc * T * p.x_stride + (size_t)nxc * T * moe_sxs(d.H) * 4);
    const size_t hb = r128((size_t)moe_h_image_bytes(T, d.I));
    p.x_bytes = (int)xb;
    struct HPlan { size_t region, h0, h1; };
    const HPlan plans[3] = {{xb + 2 * hb, xb, xb + hb},                                   // both clear of x
                            {std::max(xb, hb) + hb, std::max(xb, hb), 0},                 // buffer 0 clear of x
                            {std::max(xb, 2 * hb), 0, hb}};                               // both over x
    const int order[4][2] = {{0, 4}, {1, 3}, {2, 3}, {-1, 2}};   // (plan, fewest stages); -1: any plan
    p.ns = 0;
    for (int o = 0; o < 4 && !p.ns; ++o)
        for (int pi = 0; pi < 3 && !p.ns; ++pi) {
            if (order[o][0] >= 0 && order[o][0] != pi) continue;
            for (int ns = MOE_MAX_STAGES; ns >= order[o][1] && !p.ns; --ns)
                // a multiple of the 3 epilogue warps: they take units in turn, so
                // every buffer stays with one warp and its phases are waited on in order
                for (int nr = MOE_MAX_RED; nr >= 3; nr -= 3)
                    if (moe_decode_smem_bytes(ns, nr, (int)plans[pi].region, qc) <= (size_t)smem_optin) {
                        p.ns = ns;
                        p.nred = nr;
                        p.xh_bytes = (int)plans[pi].region;
                        p.hoff0 = (int)plans[pi].h0;
                        p.hoff1 = (int)plans[pi].h1;
                        break;
                    }
        }
    if (!p.ns) return rfx_fail(RFX_EUNSUPPORTED, "moe_ffn_forward: shapes need more shared memory than the device has");
    smem = moe_decode_smem_bytes(p.ns, p.nred, p.xh_bytes, qc);
    grid = sms;
    return RFX_OK;
}

}  // namespace rfx

extern "C" int moe_ffn_forward(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w,
                               float* y, void* ws, size_t ws_bytes, void* stream) {
    if (!layer) return rfx_fail(RFX_EINVAL, "moe_ffn_forward: null layer");
    if (T == 0) return RFX_OK;   // no token columns: nothing to do
    if (T > MOE_MAXT) return moe_ffn_prefill(layer, x, T, idx, w, y, ws, ws_bytes, stream);
    rfx::MoeParams p;
    int grid = 0;
    size_t smem = 0;
    int rc = rfx::moe_prepare(layer, x, T, idx, w, y, ws, ws_bytes, p, grid, smem);
    if (rc != RFX_OK) return rc;
    cudaError_t e = rfx::moe_decode_launch(p, grid, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("moe_ffn_forward", e);
}

// The routed step from the logits: the router launch, then the FFN launch.
// (Routing inside the FFN kernel, in its otherwise idle warps, was measured
// slower: the selection runs once per launch from a cold instruction cache
// and sits on the kernel's critical path.)
extern "C" int moe_ffn_forward_logits(const moe_layer* layer, const void* x, int T, const float* logits, int32_t* idx,
                                      float* w, float* y, void* ws, size_t ws_bytes, void* stream) {
    if (!layer) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_logits: null layer");
    if (T == 0) return RFX_OK;   // no token columns: nothing to do
    if (!logits || !idx || !w) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_logits: null pointer");
    int rc = moe_router_topk(logits, T, layer->d.E, layer->d.k, idx, w, stream);
    if (rc != RFX_OK) return rc;
    return moe_ffn_forward(layer, x, T, idx, w, y, ws, ws_bytes, stream);
}

// ------------------------------------------------------------ host buffers ---

namespace {

// Host-call scratch: the moe_ffn_forward workspace first (so rfx_ws_status
// reads its error flag at offset 0), then two sets of device copies of x and
// the logits (used in turn), the routing and y.
struct HostScratch {
    size_t ffn, x[2], logits[2], idx, w, y, total;
};

HostScratch host_scratch_layout(const moe_layer_desc& d, int T, size_t ffn_bytes) {
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    HostScratch S;
    S.ffn = 0;
    S.x[0] = up(ffn_bytes);
    S.x[1] = S.x[0] + up((size_t)T * d.H * 2);
    S.logits[0] = S.x[1] + up((size_t)T * d.H * 2);
    S.logits[1] = S.logits[0] + up((size_t)T * d.E * 4);
    S.idx = S.logits[1] + up((size_t)T * d.E * 4);
    S.w = S.idx + up((size_t)T * d.k * 4);
    S.y = S.w + up((size_t)T * d.k * 4);
    S.total = S.y + up((size_t)T * d.H * 4);
    return S;
}

// The upload stream and events of a layer, made on first use.
cudaError_t host_streams(moe_layer* L) {
    if (L->up_stream) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&L->up_stream, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&L->ev_free[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->ev_ready[i], cudaEventDisableTiming);
    }
    return e;
}

}  // namespace

extern "C" size_t moe_ffn_host_scratch_bytes(const moe_layer* layer, int T) {
    if (!layer || T < 1) return 0;
    const size_t ffn = moe_ffn_workspace_bytes(layer, T);
    if (!ffn) return 0;
    return host_scratch_layout(layer->d, T, ffn).total;
}

extern "C" int moe_ffn_forward_host(const moe_layer* layer, const void* x, const float* logits, int T, float* y,
                                    void* scratch, size_t scratch_bytes, void* stream) {
    if (!layer) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_host: null layer");
    if (T == 0) return RFX_OK;   // no token columns: nothing to do
    if (T < 1) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_host: T >= 0");
    if (!x || !logits || !y || !scratch) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_host: null pointer");
    if ((uintptr_t)scratch & 255u) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_host: scratch must be 256-byte aligned");
    const size_t ffn = moe_ffn_workspace_bytes(layer, T);
    if (!ffn) return rfx_fail(RFX_EUNSUPPORTED, "moe_ffn_forward_host: no workspace size for this layer and T");
    const moe_layer_desc& d = layer->d;
    const HostScratch S = host_scratch_layout(d, T, ffn);
    if (scratch_bytes < S.total)
        return rfx_fail(RFX_EINVAL, "moe_ffn_forward_host: scratch smaller than moe_ffn_host_scratch_bytes");
    uint8_t* b = (uint8_t*)scratch;
    int32_t* idx = (int32_t*)(b + S.idx);
    float* w = (float*)(b + S.w);
    float* yd = (float*)(b + S.y);
    cudaStream_t st = (cudaStream_t)stream;
    moe_layer* L = const_cast<moe_layer*>(layer);
    std::lock_guard<std::mutex> lock(L->host_mu);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return cuda_fail("moe_ffn_forward_host", e);
    const bool side = cap == cudaStreamCaptureStatusNone;   // a graph capture keeps everything on `stream`
    if (side) {
        e = host_streams(L);
        if (e != cudaSuccess) return cuda_fail("moe_ffn_forward_host", e);
    }
    const int s = side ? (int)(L->host_calls++ & 1u) : 0;
    void* xd = b + S.x[s];
    float* ld = (float*)(b + S.logits[s]);
    // uploads: on the side stream once the kernels of the call that used this
    // buffer set two calls ago have read it; `stream` waits for them
    cudaStream_t us = side ? L->up_stream : st;
    if (side) e = cudaStreamWaitEvent(us, L->ev_free[s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(xd, x, (size_t)T * d.H * 2, cudaMemcpyHostToDevice, us);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ld, logits, (size_t)T * d.E * 4, cudaMemcpyHostToDevice, us);
    if (side && e == cudaSuccess) e = cudaEventRecord(L->ev_ready[s], us);
    if (side && e == cudaSuccess) e = cudaStreamWaitEvent(st, L->ev_ready[s], 0);
    if (e != cudaSuccess) return cuda_fail("moe_ffn_forward_host", e);
    // decode: pinned host y that the device can address (page-locked and
    // mapped, as cudaHostAlloc / cudaHostRegister memory is under unified
    // addressing) takes the kernel's combine stores directly, with no copy
    float* ydev = nullptr;
    if (T <= MOE_MAXT) {
        cudaPointerAttributes pa{};
        if (cudaPointerGetAttributes(&pa, y) == cudaSuccess && pa.type == cudaMemoryTypeHost && pa.devicePointer)
            ydev = (float*)pa.devicePointer;
        else
            (void)cudaGetLastError();   // not an error: pageable memory takes the copy below
    }
    int rc = moe_ffn_forward_logits(layer, xd, T, ld, idx, w, ydev ? ydev : yd, b + S.ffn, S.x[0], stream);
    if (rc != RFX_OK) return rc;
    if (side) {
        e = cudaEventRecord(L->ev_free[s], st);
        if (e != cudaSuccess) return cuda_fail("moe_ffn_forward_host", e);
    }
    if (ydev) return RFX_OK;
    e = cudaMemcpyAsync(y, yd, (size_t)T * d.H * 4, cudaMemcpyDeviceToHost, st);
    return e == cudaSuccess ? RFX_OK : cuda_fail("moe_ffn_forward_host", e);
}

// ---------------------------------------------------------------- prefill ---

namespace {

const int PF_MAX_T = 1 << 16;

int prefill_check(const moe_layer* layer, int T, const char* who) {
    if (!layer) return rfx_fail(RFX_EINVAL, std::string(who) + ": null layer");
    const moe_layer_desc& d = layer->d;
    if (T < 1 || T > PF_MAX_T) return rfx_fail(RFX_EUNSUPPORTED, std::string(who) + ": 1 <= T <= 65536 tokens");
    if (d.H % 256 || d.I % 256)
        return rfx_fail(RFX_EUNSUPPORTED, std::string(who) + ": the prefill path needs H and I multiples of 256");
    return RFX_OK;
}

rfx::PfWs prefill_layout(const moe_layer* layer, int T, bool exact = false) {
    const moe_layer_desc& d = layer->d;
    return rfx::pf_ws_layout(T, d.k, d.E, d.H, d.I, exact ? 2 : 1);
}

size_t prefill_ws_bytes(const moe_layer* layer, int T, bool exact) {
    if (!layer || T < 1 || T > PF_MAX_T || layer->d.H % 256 || layer->d.I % 256) return 0;
    return prefill_layout(layer, T, exact).total;
}

int prefill_impl(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w, float* y, void* ws,
                 size_t ws_bytes, bool exact, void* stream, const char* who) {
    if (layer && T == 0) return RFX_OK;   // no tokens: nothing to do
    int rc = prefill_check(layer, T, who);
    if (rc != RFX_OK) return rc;
    const std::string W(who);
    if (!x || !idx || !w || !y || !ws) return rfx_fail(RFX_EINVAL, W + ": null pointer");
    if (!aligned16(x) || !aligned16(y) || ((uintptr_t)ws & 255u))
        return rfx_fail(RFX_EINVAL, W + ": x and y must be 16-byte and ws 256-byte aligned");
    const rfx::PfWs L = prefill_layout(layer, T, exact);
    if (ws_bytes < L.total) return rfx_fail(RFX_EINVAL, W + ": workspace smaller than its size function gives");
    int sms = 0, smem_optin = 0;
    rc = device_props(sms, smem_optin);
    if (rc != RFX_OK) return rc;
    if (std::max(rfx::pf_gemm_smem_bytes(0, exact), rfx::pf_gemm_smem_bytes(1, exact)) > (size_t)smem_optin)
        return rfx_fail(RFX_EUNSUPPORTED, W + ": the device has too little shared memory per block");
    const moe_layer_desc& d = layer->d;
    rfx::PfParams p{};
    p.H = d.H; p.I = d.I; p.E = d.E; p.k = d.k; p.T = T;
    p.mix = layer->mix_dev;
    p.fA = d.f_gate; p.fB = d.f_down;
    p.fsA = d.has_shared ? d.f_sh_gate : 2;
    p.fsB = d.has_shared ? d.f_sh_down : 2;
    p.gate = (const uint8_t*)d.gate; p.up = (const uint8_t*)d.up; p.down = (const uint8_t*)d.down;
    p.sg = (long long)d.stride_gate; p.su = (long long)d.stride_up; p.sd = (long long)d.stride_down;
    p.has_shared = d.has_shared ? 1 : 0;
    p.shg = (const uint8_t*)d.sh_gate; p.shu = (const uint8_t*)d.sh_up; p.shd = (const uint8_t*)d.sh_down;
    p.x = (const uint16_t*)x; p.idx = idx; p.wts = w; p.y = y;
    uint8_t* b = (uint8_t*)ws;
    p.ctrl = (uint32_t*)(b + L.ctrl);
    p.cnt = (int32_t*)(b + L.cnt);
    p.cnt_part = (int32_t*)(b + L.cnt_part);
    p.off = (int32_t*)(b + L.off);
    p.perm_tok = (int32_t*)(b + L.perm_tok);
    p.perm_w = (float*)(b + L.perm_w);
    p.tiles = (int4*)(b + L.tiles);
    p.xp = (uint16_t*)(b + L.xp);
    p.hp = (uint16_t*)(b + L.hp);
    p.max_tiles = L.max_tiles;
    p.exact = exact ? 1 : 0;
    p.wait_limit = rfx::debug_wait(rfx::pf_default_wait_limit());
    p.fault = rfx::debug_fault() == 3 ? 3 : 0;
    cudaError_t e = rfx::pf_launch(p, sms, (cudaStream_t)stream);
    if (e == cudaErrorInvalidValue) return rfx_fail(RFX_ECUDA, W + ": tensor-map encoding failed");
    return e == cudaSuccess ? RFX_OK : cuda_fail(who, e);
}

}  // namespace

extern "C" size_t moe_prefill_workspace_bytes(const moe_layer* layer, int T) {
    return prefill_ws_bytes(layer, T, false);
}

extern "C" int moe_ffn_prefill(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w,
                               float* y, void* ws, size_t ws_bytes, void* stream) {
    return prefill_impl(layer, x, T, idx, w, y, ws, ws_bytes, false, stream, "moe_ffn_prefill");
}

extern "C" size_t moe_prefill_workspace_bytes_ex(const moe_layer* layer, int T, int precision) {
    if (precision != RFX_PREFILL_BF16 && precision != RFX_PREFILL_EXACT) return 0;
    return prefill_ws_bytes(layer, T, precision == RFX_PREFILL_EXACT);
}

extern "C" int moe_ffn_prefill_ex(const moe_layer* layer, const void* x, int T, const int32_t* idx, const float* w,
                                  float* y, void* ws, size_t ws_bytes, int precision, void* stream) {
    if (precision != RFX_PREFILL_BF16 && precision != RFX_PREFILL_EXACT)
        return rfx_fail(RFX_EINVAL, "moe_ffn_prefill_ex: unknown precision");
    return prefill_impl(layer, x, T, idx, w, y, ws, ws_bytes, precision == RFX_PREFILL_EXACT, stream,
                        "moe_ffn_prefill_ex");
}

extern "C" int moe_prefill_view(const moe_layer* layer, int T, const void* ws, moe_prefill_ws_view* v) {
    int rc = prefill_check(layer, T, "moe_prefill_view");
    if (rc != RFX_OK) return rc;
    if (!ws || !v) return rfx_fail(RFX_EINVAL, "moe_prefill_view: null pointer");
    const rfx::PfWs L = prefill_layout(layer, T);
    const uint8_t* b = (const uint8_t*)ws;
    v->counts = (const int32_t*)(b + L.cnt);
    v->row_token = (const int32_t*)(b + L.perm_tok);
    v->row_weight = (const float*)(b + L.perm_w);
    v->h = b + L.hp;
    v->routed_rows = (int64_t)T * layer->d.k;
    v->h_rows = (int64_t)T * layer->d.k + T;
    v->h_lo = b + L.hp + (size_t)v->h_rows * layer->d.I * 2;
    return RFX_OK;
}

// ------------------------------------------------------------------ stack ---

extern "C" int moe_rms_norm_bf16(const float* y, int T, int H, void* x_next, void* stream) {
    if (T < 0 || H < 1) return rfx_fail(RFX_EINVAL, "moe_rms_norm_bf16: need T >= 0 and H >= 1");
    if (T == 0) return RFX_OK;
    if (!y || !x_next) return rfx_fail(RFX_EINVAL, "moe_rms_norm_bf16: null pointer");
    cudaError_t e = rfx::rms_bf16_launch(y, T, H, (uint16_t*)x_next, (cudaStream_t)stream);
    return e == cudaSuccess ? RFX_OK : cuda_fail("moe_rms_norm_bf16", e);
}

namespace {

// Stack workspace: one decode workspace, the routing of every layer, two
// fp32 activation buffers (layer l writes one while it reads the other).
struct StackWs {
    size_t ffn, idx, w, ybuf[2], total;
};

StackWs stack_ws_layout(const moe_layer* const* layers, int L, int T) {
    StackWs W{};
    size_t ffn = 0;
    for (int l = 0; l < L; ++l) ffn = std::max(ffn, moe_ffn_workspace_bytes(layers[l], T));
    const moe_layer_desc& d = layers[0]->d;
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    W.ffn = 0;
    W.idx = up(ffn);
    W.w = W.idx + up((size_t)L * T * d.k * 4);
    W.ybuf[0] = W.w + up((size_t)L * T * d.k * 4);
    W.ybuf[1] = W.ybuf[0] + up((size_t)T * d.H * 4);
    W.total = W.ybuf[1] + up((size_t)T * d.H * 4);
    return W;
}

int stack_check(const moe_layer* const* layers, int L, int T, const char* who) {
    if (!layers || L < 1) return rfx_fail(RFX_EINVAL, std::string(who) + ": need L >= 1 layers");
    if (T < 1 || T > MOE_MAXT) return rfx_fail(RFX_EUNSUPPORTED, std::string(who) + ": 1 <= T <= 8 token columns");
    for (int l = 0; l < L; ++l) {
        if (!layers[l]) return rfx_fail(RFX_EINVAL, std::string(who) + ": null layer");
        const moe_layer_desc& a = layers[l]->d;
        const moe_layer_desc& b = layers[0]->d;
        if (a.H != b.H || a.E != b.E || a.k != b.k)
            return rfx_fail(RFX_EINVAL, std::string(who) + ": all layers need the same H, E and k");
    }
    return RFX_OK;
}

}  // namespace

extern "C" size_t moe_stack_workspace_bytes(const moe_layer* const* layers, int L, int T) {
    if (stack_check(layers, L, T, "moe_stack_workspace_bytes") != RFX_OK) return 0;
    return stack_ws_layout(layers, L, T).total;
}

extern "C" int moe_stack_forward(const moe_layer* const* layers, int L, const float* logits, const void* x, int T,
                                 float* y, void* ws, size_t ws_bytes, void* stream) {
    if (layers && L >= 1 && T == 0) return RFX_OK;   // no token columns: nothing to do
    int rc = stack_check(layers, L, T, "moe_stack_forward");
    if (rc != RFX_OK) return rc;
    if (!logits || !x || !y || !ws) return rfx_fail(RFX_EINVAL, "moe_stack_forward: null pointer");
    if ((uintptr_t)ws & 255u) return rfx_fail(RFX_EINVAL, "moe_stack_forward: ws must be 256-byte aligned");
    const StackWs W = stack_ws_layout(layers, L, T);
    if (ws_bytes < W.total) return rfx_fail(RFX_EINVAL, "moe_stack_forward: workspace smaller than moe_stack_workspace_bytes");
    const moe_layer_desc& d = layers[0]->d;
    uint8_t* b = (uint8_t*)ws;
    int32_t* idx = (int32_t*)(b + W.idx);
    float* wts = (float*)(b + W.w);
    // the routing of all layers in one launch (it depends on the logits alone)
    rc = moe_router_topk(logits, L * T, d.E, d.k, idx, wts, stream);
    if (rc != RFX_OK) return rc;
    const float* prev = nullptr;
    for (int l = 0; l < L; ++l) {
        float* yl = l + 1 == L ? y : (float*)(b + W.ybuf[l & 1]);
        rfx::MoeParams p;
        int grid = 0;
        size_t smem = 0;
        const int32_t* il = idx + (size_t)l * T * d.k;
        const float* wl = wts + (size_t)l * T * d.k;
        rc = rfx::moe_prepare(layers[l], prev ? (const void*)prev : x, T, il, wl, yl, b + W.ffn, W.idx - W.ffn, p, grid,
                              smem);
        if (rc != RFX_OK) return rc;
        if (prev) {   // layer l > 0 takes the unit-RMS bf16 of the previous layer's y
            p.x = nullptr;
            p.xc = prev;
        }
        cudaError_t e = rfx::moe_decode_launch(p, grid, (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_fail("moe_stack_forward", e);
        prev = yl;
    }
    return RFX_OK;
}
