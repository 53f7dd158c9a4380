// Decode attention for callers that cannot allocate device memory.
//
// Some hosts embed this library where device allocation is off limits: a
// serving loop that must not call cudaMalloc once it is running (the call
// can synchronise the device and stall every stream), or a plug-in whose
// host reserves all device memory up front and never lends out more.  Such a
// caller still owns its inputs and outputs but has no way to provide the
// decode workspace.  lla_decode_attn_noalloc runs the CUDA-core decode
// kernel and its split-combine with their scratch (split partials and the
// status word) in a fixed array compiled into the library instead.
//
// The array lives in device global memory of every GPU that loads the
// library, for the life of the process.  Host code may not use the array's
// name as a device address: on the host it names a stand-in object.  The
// device address is looked up once per device with cudaGetSymbolAddress,
// with that device current, and cached: after cudaDeviceReset on a device that has served a call
// the cached address is stale, so the entry point does not support that reset (the process must
// not call this entry point on that device again).
#include <mutex>

#include "lla_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

lla_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return LLA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return LLA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LLA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" lla_status lla_decode_attn_noalloc(const lla_codec* c, const uint16_t* store, int batch, int max_tokens,
                                              int layer, int loop, const float* q, const int32_t* q_pos,
                                              const int32_t* seq_lens, float scale, float* out, void* stream) {
    if (!c || batch < 0 || max_tokens < 0 || layer < 0 || layer >= c->desc.D || loop < 0 || loop >= c->desc.T)
        return LLA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return LLA_ERR_INVALID_ARG;
    if (batch == 0) return LLA_OK;
    if (!store || !q || !q_pos || !seq_lens || !out) return LLA_ERR_INVALID_ARG;
    if (!aligned(store, 16) || !aligned(q, 16) || !aligned(out, 16) || !aligned(q_pos, 4) || !aligned(seq_lens, 4))
        return LLA_ERR_ALIGNMENT;
    // The call always runs at the automatic split count, so that is what must fit (the general
    // workspace size also reserves room for explicit split overrides, which this entry point
    // never takes).
    if (lla_simt_auto_workspace_bytes(c, batch, max_tokens) > kScratchBytes) return LLA_ERR_WORKSPACE;

    void* scratch = nullptr;
    const lla_status st = scratch_address(&scratch);
    if (st != LLA_OK) return st;

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
    call.workspace = static_cast<char*>(scratch);
    call.workspace_bytes = kScratchBytes;
    call.stream = static_cast<cudaStream_t>(stream);
    // The status word must start at zero; the split records are all rewritten by the kernel.
    LLA_CUDA_TRY(cudaMemsetAsync(scratch, 0, sizeof(lla_ws_header), call.stream));
    if (max_tokens == 0) {
        LLA_CUDA_TRY(cudaMemsetAsync(out, 0, size_t(batch) * c->desc.H * c->desc.d_head * sizeof(float), call.stream));
        return LLA_OK;
    }
    return lla_decode_simt(call, 0);
}
