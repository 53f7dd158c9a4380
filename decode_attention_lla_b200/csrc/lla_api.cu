// C ABI of the LLA library: argument validation, codec ownership, dispatch.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "lla_internal.cuh"

namespace {

uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return uint16_t((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return uint16_t(u >> 16);
}

double bf16_bits_to_double(uint16_t h) {
    uint32_t u = uint32_t(h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return double(f);
}

bool desc_valid(const lla_codec_desc* d) {
    if (!d) return false;
    if (d->D < 1 || d->T < 1 || d->H < 1 || d->d_head < 2 || (d->d_head & 1)) return false;
    if (d->r_k < 1 || d->r_v < 1 || d->max_pos < 1) return false;
    if (d->variant != 0 && d->variant != 1) return false;
    if (!(d->rope_base > 1.0f) || !isfinite(d->rope_base)) return false;
    const long long S = (long long)d->T * d->d_head * (d->variant == 1 ? d->H : 1);
    if (d->r_k > S || d->r_v > S) return false;
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

template <class T>
lla_status dev_alloc(T** p, size_t count) {
    *p = nullptr;
    if (count == 0) return LLA_OK;
    if (cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T)) != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return LLA_ERR_OOM;
    }
    return LLA_OK;
}

void codec_free(lla_codec* c) {
    if (!c) return;
    void* ptrs[] = {c->w_up_k, c->w_up_v, c->mu_k, c->mu_v, c->bias_k, c->bias_v,
                    c->w_down_k_t, c->w_down_v_t, c->rope_cos, c->rope_sin, c->phi_tiles, c->status, c->w_up_k_t,
                    c->w_up_k_bf16, c->w_up_v_bf16};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    delete c;
}

}  // namespace

int lla_num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

extern "C" {

const char* lla_status_string(lla_status s) {
    switch (s) {
        case LLA_OK: return "ok";
        case LLA_ERR_INVALID_ARG: return "invalid argument";
        case LLA_ERR_UNSUPPORTED_SHAPE: return "shape not supported by the selected kernel";
        case LLA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
        case LLA_ERR_CUDA: return "CUDA runtime error";
        case LLA_ERR_OOM: return "device out of memory";
        case LLA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char* lla_version(void) { return "lla-b200 0.1"; }

size_t lla_store_bytes(const lla_codec_desc* d, int batch, int max_tokens) {
    if (!desc_valid(d) || batch < 0 || max_tokens < 0) return 0;
    const size_t per = size_t(d->r_k + d->r_v) * (d->variant == 0 ? size_t(d->H) : 1);
    return size_t(batch) * size_t(d->D) * size_t(max_tokens) * per * 2;
}

size_t lla_paged_store_bytes(const lla_codec_desc* d, int num_pages) {
    return lla_store_bytes(d, num_pages, kPageTokens);  // a page holds kPageTokens tokens of every layer
}

lla_status lla_create_codec(lla_codec** out, const lla_codec_desc* desc, const float* w_down_k,
                            const float* w_down_v, const float* w_up_k, const float* w_up_v,
                            const float* mu_k, const float* mu_v, void* stream_) {
    if (!out) return LLA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!desc_valid(desc) || !w_down_k || !w_down_v || !w_up_k || !w_up_v || !mu_k || !mu_v)
        return LLA_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    lla_codec* c = new (std::nothrow) lla_codec();
    if (!c) return LLA_ERR_OOM;
    c->desc = *desc;
    const int D = desc->D, T = desc->T, H = desc->H, d = desc->d_head, rk = desc->r_k, rv = desc->r_v;
    const bool two_d = desc->variant == 1;
    c->S = T * d * (two_d ? H : 1);
    const int S = c->S;
    const size_t groups = two_d ? size_t(D) : size_t(D) * H;  // number of (layer[, head]) codecs
    if (cudaGetDevice(&c->device) != cudaSuccess) { delete c; return LLA_ERR_CUDA; }

    lla_status st = LLA_OK;
    const size_t nup_k = size_t(D) * T * H * d * rk, nup_v = size_t(D) * T * H * d * rv;
    const size_t nmu = groups * S;
    const int half = d / 2;
    const size_t nrope = size_t(desc->max_pos) * half;
    if ((st = dev_alloc(&c->w_up_k, nup_k)) || (st = dev_alloc(&c->w_up_v, nup_v)) ||
        (st = dev_alloc(&c->mu_k, nmu)) || (st = dev_alloc(&c->mu_v, nmu)) ||
        (st = dev_alloc(&c->bias_k, groups * rk)) || (st = dev_alloc(&c->bias_v, groups * rv)) ||
        (st = dev_alloc(&c->w_down_k_t, groups * rk * S)) || (st = dev_alloc(&c->w_down_v_t, groups * rv * S)) ||
        (st = dev_alloc(&c->rope_cos, nrope)) || (st = dev_alloc(&c->rope_sin, nrope)) ||
        (st = dev_alloc(&c->status, 4)) || (st = dev_alloc(&c->w_up_k_t, size_t(D) * T * H * (rk + 1) * d)) ||
        (st = dev_alloc(&c->w_up_k_bf16, nup_k)) || (st = dev_alloc(&c->w_up_v_bf16, nup_v))) {
        codec_free(c);
        return st;
    }

    // Host-side preparation in double precision.
    std::vector<uint16_t> wdt_k(groups * rk * S), wdt_v(groups * rv * S);
    std::vector<float> bias_k(groups * rk), bias_v(groups * rv);
    auto prep = [&](const float* wd, const float* mu, int r, std::vector<uint16_t>& wdt, std::vector<float>& bias) {
        for (size_t g = 0; g < groups; ++g) {
            const float* W = wd + g * size_t(S) * r;
            const float* m = mu + g * size_t(S);
            for (int a = 0; a < r; ++a) {
                double acc = 0.0;
                uint16_t* row = wdt.data() + (g * r + a) * size_t(S);
                for (int k = 0; k < S; ++k) {
                    const uint16_t w16 = f32_to_bf16_rne(W[size_t(k) * r + a]);
                    row[k] = w16;
                    acc += double(m[k]) * bf16_bits_to_double(w16);
                }
                bias[g * r + a] = float(acc);  // b = mu W_down, from the bf16 W_down the kernel uses
            }
        }
    };
    prep(w_down_k, mu_k, rk, wdt_k, bias_k);
    prep(w_down_v, mu_v, rv, wdt_v, bias_v);
    std::vector<float> rc(nrope), rs(nrope);
    for (int i = 0; i < half; ++i) {
        const double theta = pow(double(desc->rope_base), -2.0 * i / d);
        for (int pos = 0; pos < desc->max_pos; ++pos) {
            const double ang = double(pos) * theta;
            rc[size_t(pos) * half + i] = float(cos(ang));
            rs[size_t(pos) * half + i] = float(sin(ang));
        }
    }
    // W^K_up,t transposed, mu^K_t appended as row r_k: [(layer, head, loop) slot][r_k + 1][d]
    std::vector<float> wupt(size_t(D) * T * H * (rk + 1) * d);
    for (int l = 0; l < D; ++l)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const size_t g = two_d ? (size_t(l) * T + t) * H + h : (size_t(l) * H + h) * T + t;
                const float* W = w_up_k + g * size_t(d) * rk;
                const float* m = two_d ? mu_k + size_t(l) * S + (size_t(t) * H + h) * d
                                       : mu_k + (size_t(l) * H + h) * S + size_t(t) * d;
                float* o = wupt.data() + g * size_t(rk + 1) * d;
                for (int n = 0; n < rk; ++n)
                    for (int i = 0; i < d; ++i) o[size_t(n) * d + i] = W[size_t(i) * rk + n];
                for (int i = 0; i < d; ++i) o[size_t(rk) * d + i] = m[i];
            }
    std::vector<uint16_t> wup16_k(nup_k), wup16_v(nup_v);
    for (size_t i = 0; i < nup_k; ++i) wup16_k[i] = f32_to_bf16_rne(w_up_k[i]);
    for (size_t i = 0; i < nup_v; ++i) wup16_v[i] = f32_to_bf16_rne(w_up_v[i]);
    bool ok = cudaMemcpyAsync(c->w_up_k_t, wupt.data(), wupt.size() * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_up_k_bf16, wup16_k.data(), nup_k * 2, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_up_v_bf16, wup16_v.data(), nup_v * 2, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_up_k, w_up_k, nup_k * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_up_v, w_up_v, nup_v * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->mu_k, mu_k, nmu * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->mu_v, mu_v, nmu * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->bias_k, bias_k.data(), bias_k.size() * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->bias_v, bias_v.data(), bias_v.size() * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_down_k_t, wdt_k.data(), wdt_k.size() * 2, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->w_down_v_t, wdt_v.data(), wdt_v.size() * 2, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->rope_cos, rc.data(), rc.size() * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemcpyAsync(c->rope_sin, rs.data(), rs.size() * 4, cudaMemcpyHostToDevice, stream) == cudaSuccess &&
              cudaMemsetAsync(c->status, 0, 4 * sizeof(uint32_t), stream) == cudaSuccess;
    if (ok) ok = lla_build_phi_tiles(c, stream) == LLA_OK;
    if (ok) ok = cudaStreamSynchronize(stream) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        codec_free(c);
        return LLA_ERR_CUDA;
    }
    *out = c;
    return LLA_OK;
}

lla_status lla_destroy_codec(lla_codec* c) {
    if (!c) return LLA_OK;
    cudaDeviceSynchronize();
    codec_free(c);
    return LLA_OK;
}

lla_status lla_codec_get_desc(const lla_codec* c, lla_codec_desc* out) {
    if (!c || !out) return LLA_ERR_INVALID_ARG;
    *out = c->desc;
    return LLA_OK;
}

lla_status lla_encode(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                      const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch,
                      int max_tokens, void* stream) {
    if (!c || n < 0 || batch < 0 || max_tokens < 0) return LLA_ERR_INVALID_ARG;
    if (layer_begin < 0 || num_layers < 1 || layer_begin + num_layers > c->desc.D) return LLA_ERR_INVALID_ARG;
    if (n == 0) return LLA_OK;
    if (!x || !seq_idx || !tok_idx || !store) return LLA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(store) || !aligned4(seq_idx) || !aligned4(tok_idx)) return LLA_ERR_ALIGNMENT;
    return lla_encode_launch(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch, max_tokens,
                             static_cast<cudaStream_t>(stream));
}

lla_status lla_encode_paged(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                            const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* pool, int num_pages,
                            const int32_t* block_table, int max_pages, int batch, void* stream) {
    if (!c || n < 0 || batch < 0 || num_pages < 1 || max_pages < 1) return LLA_ERR_INVALID_ARG;
    if (max_pages > (1 << 30) / kPageTokens) return LLA_ERR_INVALID_ARG;
    if (layer_begin < 0 || num_layers < 1 || layer_begin + num_layers > c->desc.D) return LLA_ERR_INVALID_ARG;
    if (n == 0) return LLA_OK;
    if (!x || !seq_idx || !tok_idx || !pool || !block_table) return LLA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(pool) || !aligned4(seq_idx) || !aligned4(tok_idx) || !aligned4(block_table))
        return LLA_ERR_ALIGNMENT;
    lla_store_map smap;
    smap.table = block_table;
    smap.max_pages = max_pages;
    smap.num_pages = num_pages;
    return lla_encode_launch(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, pool, batch,
                             max_pages * kPageTokens, static_cast<cudaStream_t>(stream), smap);
}

size_t lla_decode_workspace_bytes(const lla_codec* c, int batch, int max_tokens) {
    if (!c || batch < 0 || max_tokens < 0) return 0;
    size_t a = lla_simt_workspace_bytes(c, batch, max_tokens);
    if (lla_tc_supported(c)) {
        const size_t b = lla_tc_workspace_bytes(c, batch, max_tokens);
        if (b > a) a = b;
    }
    return a;
}

static lla_status decode_common(int want_variant, const lla_codec* c, const uint16_t* store, int batch,
                                int max_tokens, int layer, int loop, const float* q, const int32_t* q_pos,
                                const int32_t* seq_lens, float scale, float* out, void* workspace,
                                size_t workspace_bytes, const lla_decode_opts* opts, void* stream,
                                const float* k_self = nullptr, const float* v_self = nullptr,
                                const lla_store_map& smap = lla_store_map()) {
    if (!c || c->desc.variant != want_variant) return LLA_ERR_INVALID_ARG;
    if (batch < 0 || max_tokens < 0 || layer < 0 || layer >= c->desc.D || loop < 0 || loop >= c->desc.T)
        return LLA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LLA_ERR_INVALID_ARG;
    if (batch == 0) return LLA_OK;
    if (!store || !q || !q_pos || !seq_lens || !out) return LLA_ERR_INVALID_ARG;
    if (!workspace) return LLA_ERR_WORKSPACE;
    if (!aligned16(store) || !aligned16(q) || !aligned16(out) || !aligned16(workspace) || !aligned4(q_pos) ||
        !aligned4(seq_lens))
        return LLA_ERR_ALIGNMENT;
    if ((k_self == nullptr) != (v_self == nullptr)) return LLA_ERR_INVALID_ARG;
    if (k_self && (!aligned16(k_self) || !aligned16(v_self))) return LLA_ERR_ALIGNMENT;
    if (workspace_bytes < lla_decode_workspace_bytes(c, batch, max_tokens)) return LLA_ERR_WORKSPACE;
    const int impl = opts ? opts->impl : 0;
    const int num_ctas = opts ? opts->num_ctas : 0;
    if (impl < 0 || impl > 2 || num_ctas < 0) return LLA_ERR_INVALID_ARG;

    lla_decode_call call;
    call.codec = c;
    call.store = store;
    call.batch = batch;
    call.max_tokens = max_tokens;
    call.layer = layer;
    call.loop = loop;
    call.q = q;
    call.q_pos = q_pos;
    call.seq_lens = seq_lens;
    call.scale = scale;
    call.out = out;
    call.workspace = static_cast<char*>(workspace);
    call.workspace_bytes = workspace_bytes;
    call.stream = static_cast<cudaStream_t>(stream);
    if (opts) {
        call.ev_begin = static_cast<cudaEvent_t>(opts->ev_begin);
        call.ev_end = static_cast<cudaEvent_t>(opts->ev_end);
    }
    call.k_self = k_self;
    call.v_self = v_self;
    call.smap = smap;
    LLA_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(lla_ws_header), call.stream));
    if (max_tokens == 0) {
        // no cached token: the softmax is empty (zero output) or the self slot alone (its value)
        const size_t bytes = size_t(batch) * c->desc.H * c->desc.d_head * 4;
        if (v_self) LLA_CUDA_TRY(cudaMemcpyAsync(out, v_self, bytes, cudaMemcpyDeviceToDevice, call.stream));
        else LLA_CUDA_TRY(cudaMemsetAsync(out, 0, bytes, call.stream));
        return LLA_OK;
    }
    const bool tc_ok = lla_tc_supported(c);
    if (impl == 2 && !tc_ok) return LLA_ERR_UNSUPPORTED_SHAPE;
    if (impl == 2 || (impl == 0 && tc_ok)) return lla_decode_tc(call, num_ctas);
    return lla_decode_simt(call, num_ctas);
}

lla_status lla_decode_attn(const lla_codec* c, const uint16_t* store, int batch, int max_tokens, int layer,
                           int loop, const float* q, const int32_t* q_pos, const int32_t* seq_lens,
                           float scale, float* out, void* workspace, size_t workspace_bytes, void* stream) {
    return decode_common(0, c, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, workspace,
                         workspace_bytes, nullptr, stream);
}

lla_status lla_decode_attn_2d(const lla_codec* c, const uint16_t* store, int batch, int max_tokens, int layer,
                              int loop, const float* q, const int32_t* q_pos, const int32_t* seq_lens,
                              float scale, float* out, void* workspace, size_t workspace_bytes, void* stream) {
    return decode_common(1, c, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, workspace,
                         workspace_bytes, nullptr, stream);
}

lla_status lla_decode_attn_ex(const lla_codec* c, const uint16_t* store, int batch, int max_tokens, int layer,
                              int loop, const float* q, const int32_t* q_pos, const int32_t* seq_lens,
                              float scale, float* out, void* workspace, size_t workspace_bytes,
                              const lla_decode_opts* opts, void* stream) {
    if (!c) return LLA_ERR_INVALID_ARG;
    return decode_common(c->desc.variant, c, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out,
                         workspace, workspace_bytes, opts, stream);
}

lla_status lla_decode_attn_self(const lla_codec* c, const uint16_t* store, int batch, int max_tokens, int layer,
                                int loop, const float* q, const int32_t* q_pos, const int32_t* seq_lens,
                                const float* k_self, const float* v_self, float scale, float* out,
                                void* workspace, size_t workspace_bytes, const lla_decode_opts* opts,
                                void* stream) {
    if (!c) return LLA_ERR_INVALID_ARG;
    if (batch > 0 && (!k_self || !v_self)) return LLA_ERR_INVALID_ARG;
    return decode_common(c->desc.variant, c, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out,
                         workspace, workspace_bytes, opts, stream, k_self, v_self);
}

lla_status lla_decode_attn_paged(const lla_codec* c, const uint16_t* pool, int num_pages, const int32_t* block_table,
                                 int max_pages, int batch, int layer, int loop, const float* q, const int32_t* q_pos,
                                 const int32_t* seq_lens, const float* k_self, const float* v_self, float scale,
                                 float* out, void* workspace, size_t workspace_bytes, const lla_decode_opts* opts,
                                 void* stream) {
    if (!c || num_pages < 1 || max_pages < 1 || max_pages > (1 << 30) / kPageTokens) return LLA_ERR_INVALID_ARG;
    if (batch > 0 && !block_table) return LLA_ERR_INVALID_ARG;
    if (block_table && !aligned4(block_table)) return LLA_ERR_ALIGNMENT;
    lla_store_map smap;
    smap.table = block_table;
    smap.max_pages = max_pages;
    smap.num_pages = num_pages;
    return decode_common(c->desc.variant, c, pool, batch, max_pages * kPageTokens, layer, loop, q, q_pos, seq_lens,
                         scale, out, workspace, workspace_bytes, opts, stream, k_self, v_self, smap);
}

size_t lla_full_decode_workspace_bytes(int H, int d_head, int batch) {
    if (H < 1 || d_head != 128 || batch < 0) return 0;
    return lla_full_workspace_bytes(H, batch);
}

lla_status lla_full_decode_attn(int H, int d_head, float rope_base, const uint16_t* k_cache, const uint16_t* v_cache,
                                long long seq_stride, int batch, int max_tokens, const float* q,
                                const int32_t* q_pos, const int32_t* seq_lens, float scale, float* out,
                                void* workspace, size_t workspace_bytes, int num_ctas, void* stream) {
    if (H < 1 || batch < 0 || max_tokens < 0 || num_ctas < 0 || !isfinite(scale) || !(rope_base > 0.f))
        return LLA_ERR_INVALID_ARG;
    if (d_head != 128) return LLA_ERR_UNSUPPORTED_SHAPE;
    if (batch == 0) return LLA_OK;
    if (!k_cache || !v_cache || !q || !q_pos || !seq_lens || !out) return LLA_ERR_INVALID_ARG;
    if (!workspace) return LLA_ERR_WORKSPACE;
    if (seq_stride < (long long)max_tokens * H * d_head || seq_stride % 8 != 0) return LLA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out) || !aligned16(workspace) ||
        !aligned4(q_pos) || !aligned4(seq_lens))
        return LLA_ERR_ALIGNMENT;
    if (workspace_bytes < lla_full_workspace_bytes(H, batch)) return LLA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (max_tokens == 0) {
        LLA_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(lla_ws_header), st));
        LLA_CUDA_TRY(cudaMemsetAsync(out, 0, size_t(batch) * H * d_head * 4, st));
        return LLA_OK;
    }
    return lla_full_decode(H, rope_base, k_cache, v_cache, seq_stride, batch, max_tokens, q, q_pos, seq_lens, scale,
                           out, workspace, workspace_bytes, num_ctas, st);
}

size_t lla_fit_codec_workspace_bytes(int problems, int n, int S, int r) {
    if (problems < 1 || problems > 65535 || n < 1 || S < 1 || r < 1 || r > (n < S ? n : S) ||
        (n < S ? n : S) > 32768 || !lla_fit_shape_ok(n, S, r))
        return 0;
    return lla_fit_workspace_bytes_impl(problems, n, S, r);
}

lla_status lla_fit_codec(int problems, int n, int S, int r, const float* X, float* mu, float* w_down, float* sigma,
                         int iters, void* workspace, size_t workspace_bytes, void* stream) {
    if (problems < 0 || n < 1 || S < 1 || r < 1 || iters < 0) return LLA_ERR_INVALID_ARG;
    const int m = n < S ? n : S;
    if (r > m) return LLA_ERR_INVALID_ARG;
    if (m > 32768 || problems > 65535 || !lla_fit_shape_ok(n, S, r)) return LLA_ERR_UNSUPPORTED_SHAPE;
    if (problems == 0) return LLA_OK;
    if (!X || !mu || !w_down) return LLA_ERR_INVALID_ARG;
    if (!workspace) return LLA_ERR_WORKSPACE;
    if (!aligned4(X) || !aligned4(mu) || !aligned4(w_down) || (sigma && !aligned4(sigma)) || !aligned16(workspace))
        return LLA_ERR_ALIGNMENT;
    if (workspace_bytes < lla_fit_workspace_bytes_impl(problems, n, S, r)) return LLA_ERR_WORKSPACE;
    return lla_fit(problems, n, S, r, X, mu, w_down, sigma, iters == 0 ? 24 : iters, workspace,
                   static_cast<cudaStream_t>(stream));
}

lla_status lla_reconstruct_cache(const lla_codec* c, const uint16_t* store, int batch, int max_tokens, int layer,
                                 int loop, const int32_t* seq_lens, uint16_t* k_cache, uint16_t* v_cache,
                                 long long seq_stride, int cache_tokens, int impl, void* stream) {
    if (!c || batch < 0 || max_tokens < 0 || layer < 0 || layer >= c->desc.D || loop < 0 || loop >= c->desc.T)
        return LLA_ERR_INVALID_ARG;
    if (impl < 0 || impl > 2 || max_tokens > c->desc.max_pos || cache_tokens < max_tokens) return LLA_ERR_INVALID_ARG;
    if (batch == 0 || max_tokens == 0) return LLA_OK;
    if (!store || !seq_lens || !k_cache || !v_cache) return LLA_ERR_INVALID_ARG;
    const long long seq_elems = (long long)c->desc.H * cache_tokens * c->desc.d_head;
    if (seq_stride < seq_elems || seq_stride % 8 != 0) return LLA_ERR_INVALID_ARG;
    if (!aligned16(store) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned4(seq_lens))
        return LLA_ERR_ALIGNMENT;
    if (impl == 2 && !lla_reconstruct_tc_supported(c)) return LLA_ERR_UNSUPPORTED_SHAPE;
    lla_reconstruct_call rc;
    rc.codec = c;
    rc.store = store;
    rc.batch = batch;
    rc.max_tokens = max_tokens;
    rc.layer = layer;
    rc.loop = loop;
    rc.seq_lens = seq_lens;
    rc.k_cache = k_cache;
    rc.v_cache = v_cache;
    rc.seq_stride = seq_stride;
    rc.cache_tokens = cache_tokens;
    rc.stream = static_cast<cudaStream_t>(stream);
    return lla_reconstruct_launch(rc, impl);
}

lla_status lla_workspace_flags(const void* workspace, uint32_t* flags, void* stream) {
    if (!workspace || !flags) return LLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LLA_CUDA_TRY(cudaMemcpyAsync(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
    LLA_CUDA_TRY(cudaStreamSynchronize(s));
    return LLA_OK;
}

}  // extern "C"
