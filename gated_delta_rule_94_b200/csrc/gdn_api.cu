// gdn_api.cu -- host side of the libgdn C ABI (include/gdn.h): argument
// validation, workspace sizing, kernel selection and launch on the caller's
// stream.  Nothing here allocates device memory or synchronizes, except
// gdn_read_device_status, which is documented to synchronize.
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gdn.h"

// The library's device status word: kernels OR in StatusBits when they give up
// a bounded wait; gdn_read_device_status reads and clears it.
__device__ unsigned gdn_device_status_word = 0u;

namespace {

unsigned* status_word_ptr() {
    // One device address per current device, looked up once per device
    // ordinal under a lock (calls may come from several host threads).  A
    // failed lookup clears the runtime's last-error state so that it is not
    // reported later by an unrelated call.
    static std::mutex mu;
    static unsigned* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, gdn_device_status_word) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        cache[dev] = static_cast<unsigned*>(ptr);
    }
    return cache[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

std::atomic<unsigned long long> g_launches{0};

bool supported_dim(int d) { return d == 64 || d == 128; }

size_t elem_size(gdn_dtype dt) { return dt == GDN_BF16 ? 2 : 4; }

}  // namespace

extern "C" {

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_ERR_UNKNOWN";
}

int gdn_abi_version(void) { return 1; }

unsigned long long gdn_kernel_launch_count(void) { return g_launches.load(); }

const char* gdn_chunk_fwd_kernel_name(int Dk, int Dv, gdn_gate gate_kind, gdn_dtype dtype) {
    if (!supported_dim(Dk) || !supported_dim(Dv)) return nullptr;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return nullptr;
    if (dtype == GDN_BF16 && gdn::chunk_fwd_tc_supported(Dk, Dv, gate_kind))
        return "chunk_prep_kernel,chunk_chain_kernel";
    if (dtype == GDN_BF16 || dtype == GDN_F32) return "chunk_fwd_simt_kernel";
    return nullptr;
}

size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                     gdn_dtype dtype, gdn_gate gate_kind) {
    if (B < 0 || T < 0 || H < 0) return (size_t)-1;
    if (!supported_dim(Dk) || !supported_dim(Dv) || chunk != 64) return (size_t)-1;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return (size_t)-1;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return (size_t)-1;
    if (dtype == GDN_BF16 && gdn::chunk_fwd_tc_supported(Dk, Dv, gate_kind))
        return gdn::chunk_fwd_tc_workspace_bytes(B, T, H, gate_kind);
    return 0;
}

size_t gdn_chunk_fwd_workspace_min_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                         gdn_dtype dtype, gdn_gate gate_kind) {
    if (B < 0 || T < 0 || H < 0) return (size_t)-1;
    if (!supported_dim(Dk) || !supported_dim(Dv) || chunk != 64) return (size_t)-1;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return (size_t)-1;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return (size_t)-1;
    if (dtype == GDN_BF16 && gdn::chunk_fwd_tc_supported(Dk, Dv, gate_kind))
        return gdn::chunk_fwd_tc_workspace_min_bytes(B, T, H, gate_kind);
    return 0;
}

gdn_status gdn_chunk_fwd_plan(int B, int T, int H, int Dk, int Dv, int chunk, gdn_dtype dtype,
                              gdn_gate gate_kind, size_t workspace_bytes, int* waves,
                              int* chunks_per_wave, int* segments) {
    if (!waves || !chunks_per_wave || !segments) return GDN_ERR_INVALID_ARG;
    const size_t least =
        gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dv, chunk, dtype, gate_kind);
    if (least == (size_t)-1) {
        if (B < 0 || T < 0 || H < 0 || (dtype != GDN_BF16 && dtype != GDN_F32) ||
            gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM)
            return GDN_ERR_INVALID_ARG;
        return GDN_ERR_UNSUPPORTED;
    }
    if (workspace_bytes < least) return GDN_ERR_WORKSPACE;
    const int NC = (T + 63) / 64;
    *waves = B * H > 0 && NC > 0 ? 1 : 0;
    *chunks_per_wave = NC;
    *segments = *waves;
    if (least > 0)   // the tensor-core path
        gdn::chunk_fwd_tc_plan(B, T, H, gate_kind, workspace_bytes, waves, chunks_per_wave,
                               segments);
    return GDN_OK;
}

}  // extern "C"

namespace {

// The chunk forward, with the write key kw (null: kw = k).
gdn_status chunk_fwd_impl(const void* q, const void* k, const void* kw, const void* v,
                          const void* beta, const void* g, gdn_gate gate_kind,
                          const float* initial_state, void* o, float* final_state, int B, int T,
                          int H, int Dk, int Dv, int chunk, gdn_dtype dtype, void* workspace,
                          size_t workspace_bytes, gdn_stream_t stream) {
    if (B < 0 || T < 0 || H < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(Dk) || !supported_dim(Dv) || chunk != 64) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)B * T > INT32_MAX || (int64_t)B * H > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return GDN_OK;
    const bool need_tokens = T > 0;
    if (need_tokens && (!q || !k || !v || !beta || !o)) return GDN_ERR_INVALID_ARG;
    if (need_tokens && (gate_kind == GDN_GATE_NONE) != (g == nullptr)) return GDN_ERR_INVALID_ARG;
    // a separate write key runs on the tensor-core path only
    if (kw && !(dtype == GDN_BF16 && gdn::chunk_fwd_tc_supported(Dk, Dv, gate_kind)))
        return GDN_ERR_UNSUPPORTED;
    const void* ptrs[] = {q, k, kw, v, beta, g, initial_state, o, final_state, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t ntok = (size_t)B * T * H;
    const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
    if (final_state) {
        const size_t gbytes = gate_kind == GDN_GATE_PER_DIM ? ntok * Dk * es
                              : gate_kind == GDN_GATE_SCALAR ? ntok * es : 0;
        if (overlaps(final_state, state_bytes, q, ntok * Dk * es) ||
            overlaps(final_state, state_bytes, k, ntok * Dk * es) ||
            overlaps(final_state, state_bytes, kw, ntok * Dk * es) ||
            overlaps(final_state, state_bytes, v, ntok * Dv * es) ||
            overlaps(final_state, state_bytes, beta, ntok * es) ||
            overlaps(final_state, state_bytes, g, gbytes) ||
            overlaps(final_state, state_bytes, o, ntok * Dv * es))
            return GDN_ERR_INVALID_ARG;
        if (initial_state && initial_state != final_state &&
            overlaps(final_state, state_bytes, initial_state, state_bytes))
            return GDN_ERR_INVALID_ARG;
    }
    if (need_tokens && initial_state && overlaps(o, ntok * Dv * es, initial_state, state_bytes))
        return GDN_ERR_INVALID_ARG;
    if (need_tokens && kw && overlaps(o, ntok * Dv * es, kw, ntok * Dk * es)) return GDN_ERR_INVALID_ARG;
    const size_t ws_need = gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dv, chunk, dtype, gate_kind);
    if (ws_need > 0 && (workspace_bytes < ws_need || !workspace)) return GDN_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        // No tokens: the final state is the initial state (or zero).
        if (!final_state) return GDN_OK;
        cudaError_t e = initial_state
                            ? (initial_state == final_state
                                   ? cudaSuccess
                                   : cudaMemcpyAsync(final_state, initial_state, state_bytes,
                                                     cudaMemcpyDeviceToDevice, s))
                            : cudaMemsetAsync(final_state, 0, state_bytes, s);
        return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }

    gdn::ChunkParams p{};
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.g = g; p.kw = kw;
    p.s0 = initial_state; p.o = o; p.s_out = final_state;
    p.B = B; p.T = T; p.H = H; p.Dk = Dk; p.Dv = Dv;
    p.status = status_word_ptr();
    p.ws = static_cast<uint8_t*>(workspace);
    p.cw = 0;
    p.chunk0 = 0;
    p.nchunks = 0;
    p.ws_chunk = 0;
    if (!p.status) return GDN_ERR_CUDA;
    cudaError_t e;
    int launches = 1;
    if (dtype == GDN_BF16 && gdn::chunk_fwd_tc_supported(Dk, Dv, gate_kind))
        e = gdn::launch_chunk_fwd_tc(p, gate_kind, workspace_bytes, s, &launches);
    else
        e = gdn::launch_chunk_fwd_simt(p, gate_kind, dtype == GDN_BF16, s);
    g_launches.fetch_add((unsigned long long)launches);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const void* beta,
                         const void* g, gdn_gate gate_kind, const float* initial_state,
                         void* o, float* final_state, int B, int T, int H, int Dk, int Dv,
                         int chunk, gdn_dtype dtype, void* workspace, size_t workspace_bytes,
                         gdn_stream_t stream) {
    return chunk_fwd_impl(q, k, nullptr, v, beta, g, gate_kind, initial_state, o, final_state,
                          B, T, H, Dk, Dv, chunk, dtype, workspace, workspace_bytes, stream);
}

gdn_status gdn_chunk_fwd_wk(const void* q, const void* k, const void* k_write, const void* v,
                            const void* beta, const void* g, gdn_gate gate_kind,
                            const float* initial_state, void* o, float* final_state, int B,
                            int T, int H, int Dk, int Dv, int chunk, gdn_dtype dtype,
                            void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    return chunk_fwd_impl(q, k, k_write, v, beta, g, gate_kind, initial_state, o, final_state,
                          B, T, H, Dk, Dv, chunk, dtype, workspace, workspace_bytes, stream);
}

size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                     gdn_dtype dtype, gdn_gate gate_kind) {
    if (B < 0 || T < 0 || H < 0) return (size_t)-1;
    if (Dk != 128 || Dv != 128 || chunk != 64 || dtype != GDN_BF16) return (size_t)-1;
    if (gate_kind != GDN_GATE_NONE && gate_kind != GDN_GATE_SCALAR) return (size_t)-1;
    return gdn::chunk_bwd_workspace_bytes(B, T, H);
}

gdn_status gdn_chunk_bwd(const void* q, const void* k, const void* v, const void* beta,
                         const void* g, gdn_gate gate_kind, const float* initial_state,
                         const void* d_o, const float* d_final_state, float* dq, float* dk,
                         float* dv, float* dbeta, float* dg, float* d_initial_state, int B,
                         int T, int H, int Dk, int Dv, int chunk, gdn_dtype dtype,
                         void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (B < 0 || T < 0 || H < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return GDN_ERR_INVALID_ARG;
    if (Dk != 128 || Dv != 128 || chunk != 64 || dtype != GDN_BF16 ||
        gate_kind == GDN_GATE_PER_DIM)
        return GDN_ERR_UNSUPPORTED;
    if ((int64_t)B * T > INT32_MAX || (int64_t)B * H > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return GDN_OK;
    const bool tokens = T > 0;
    if (tokens && (!q || !k || !v || !beta || !d_o || !dq || !dk || !dv || !dbeta))
        return GDN_ERR_INVALID_ARG;
    if (tokens && (gate_kind == GDN_GATE_NONE) != (g == nullptr)) return GDN_ERR_INVALID_ARG;
    if (tokens && gate_kind == GDN_GATE_SCALAR && !dg) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, g, initial_state, d_o, d_final_state, dq, dk, dv,
                          dbeta, dg, d_initial_state, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t ntok = (size_t)B * T * H;
    const size_t sb = (size_t)B * H * Dk * Dv * sizeof(float);
    // every output must be clear of every input and of the other outputs
    const void* outs[] = {dq, dk, dv, dbeta, dg, d_initial_state};
    const size_t outn[] = {ntok * Dk * 4, ntok * Dk * 4, ntok * Dv * 4, ntok * 4,
                           g ? ntok * 4 : 0, sb};
    const void* ins[] = {q, k, v, beta, g, initial_state, d_o, d_final_state};
    const size_t inn[] = {ntok * Dk * 2, ntok * Dk * 2, ntok * Dv * 2, ntok * 2, ntok * 2, sb,
                          ntok * Dv * 2, sb};
    for (int i = 0; i < 6; ++i) {
        for (int j = 0; j < 8; ++j)
            if (overlaps(outs[i], outn[i], ins[j], inn[j])) return GDN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 6; ++j)
            if (overlaps(outs[i], outn[i], outs[j], outn[j])) return GDN_ERR_INVALID_ARG;
    }
    const size_t need = gdn::chunk_bwd_workspace_bytes(B, T, H);
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {   // no tokens: the final state is the initial state
        if (!d_initial_state) return GDN_OK;
        const cudaError_t e = d_final_state
            ? cudaMemcpyAsync(d_initial_state, d_final_state, sb, cudaMemcpyDeviceToDevice, s)
            : cudaMemsetAsync(d_initial_state, 0, sb, s);
        return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    }
    gdn::ChunkParams pf{};
    pf.q = q; pf.k = k; pf.v = v; pf.beta = beta; pf.g = g;
    pf.s0 = initial_state; pf.B = B; pf.T = T; pf.H = H; pf.Dk = Dk; pf.Dv = Dv;
    pf.status = status_word_ptr();
    if (!pf.status) return GDN_ERR_CUDA;
    gdn::BwdParams pb{};
    pb.q = q; pb.k = k; pb.v = v; pb.beta = beta; pb.g = g; pb.dO = d_o; pb.dS = d_final_state;
    pb.dq = dq; pb.dk = dk; pb.dv = dv; pb.dbeta = dbeta; pb.dg = dg; pb.dS0 = d_initial_state;
    pb.B = B; pb.T = T; pb.H = H;
    pb.status = pf.status;
    int launches = 0;
    const cudaError_t e = gdn::launch_chunk_bwd(pf, pb, gate_kind,
                                                static_cast<uint8_t*>(workspace), workspace_bytes,
                                                s, &launches);
    g_launches.fetch_add((unsigned long long)launches);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_osdn_precondition_workspace_bytes(int B, int T, int H, int Dk) {
    if (B < 0 || T < 0 || H < 0 || !supported_dim(Dk)) return (size_t)-1;
    return gdn::osdn_precondition_workspace_bytes(B, T, H, Dk);
}

gdn_status gdn_osdn_precondition(const void* k, const void* beta, const void* r, float eta,
                                 const float* d0, void* k_write, float* d_final, int B, int T,
                                 int H, int Dk, gdn_dtype dtype, void* workspace,
                                 size_t workspace_bytes, gdn_stream_t stream) {
    if (B < 0 || T < 0 || H < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (!(eta == eta) || eta > 3.0e38f || eta < -3.0e38f) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(Dk)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)B * T > INT32_MAX || (int64_t)B * H > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return GDN_OK;
    if (T > 0 && (!k || !beta || !k_write)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {k, beta, r, d0, k_write, d_final, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t ntok = (size_t)B * T * H;
    const size_t dbytes = (size_t)B * H * Dk * sizeof(float);
    const size_t need = gdn::osdn_precondition_workspace_bytes(B, T, H, Dk);
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    const void* others[] = {k, beta, r, d0, k_write, d_final};
    const size_t othern[] = {ntok * Dk * es, ntok * es, ntok * es, dbytes, ntok * Dk * es, dbytes};
    for (int i = 0; i < 6; ++i)
        if (overlaps(workspace, need, others[i], othern[i])) return GDN_ERR_INVALID_ARG;
    if (overlaps(k_write, ntok * Dk * es, k, ntok * Dk * es) ||
        overlaps(k_write, ntok * Dk * es, beta, ntok * es) ||
        overlaps(k_write, ntok * Dk * es, r, ntok * es) ||
        overlaps(k_write, ntok * Dk * es, d0, dbytes) ||
        overlaps(k_write, ntok * Dk * es, d_final, dbytes) ||
        overlaps(d_final, dbytes, k, ntok * Dk * es) ||
        overlaps(d_final, dbytes, beta, ntok * es) ||
        overlaps(d_final, dbytes, r, ntok * es))
        return GDN_ERR_INVALID_ARG;
    if (d0 && d_final && d0 != d_final && overlaps(d0, dbytes, d_final, dbytes))
        return GDN_ERR_INVALID_ARG;
    if (T == 0 && !d_final) return GDN_OK;
    gdn::OsdnParams p;
    p.k = k; p.beta = beta; p.r = r; p.kw = k_write; p.d0 = d0; p.d_out = d_final;
    p.eta = eta; p.B = B; p.T = T; p.H = H;
    int launches = 0;
    cudaError_t e = gdn::launch_osdn_precondition(p, Dk, dtype == GDN_BF16,
                                                  static_cast<uint8_t*>(workspace),
                                                  reinterpret_cast<cudaStream_t>(stream), &launches);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    g_launches.fetch_add((unsigned long long)launches);
    return GDN_OK;
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, const void* beta,
                           const void* g, gdn_gate gate_kind, float* state, void* o, int N,
                           int H, int Dk, int Dv, gdn_dtype dtype, gdn_stream_t stream) {
    if (N < 0 || H < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (gate_kind < GDN_GATE_NONE || gate_kind > GDN_GATE_PER_DIM) return GDN_ERR_INVALID_ARG;
    if (!supported_dim(Dk) || !supported_dim(Dv)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)N * H > INT32_MAX) return GDN_ERR_UNSUPPORTED;
    if (N == 0 || H == 0) return GDN_OK;
    if (!q || !k || !v || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if ((gate_kind == GDN_GATE_NONE) != (g == nullptr)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, g, state, o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t nh = (size_t)N * H;
    const size_t state_bytes = nh * Dk * Dv * sizeof(float);
    const size_t gbytes = gate_kind == GDN_GATE_PER_DIM ? nh * Dk * es
                          : gate_kind == GDN_GATE_SCALAR ? nh * es : 0;
    if (overlaps(state, state_bytes, o, nh * Dv * es) ||
        overlaps(state, state_bytes, q, nh * Dk * es) ||
        overlaps(state, state_bytes, k, nh * Dk * es) ||
        overlaps(state, state_bytes, v, nh * Dv * es) ||
        overlaps(state, state_bytes, beta, nh * es) ||
        overlaps(state, state_bytes, g, gbytes))
        return GDN_ERR_INVALID_ARG;

    gdn::DecodeParams p;
    p.q = q; p.k = k; p.v = v; p.beta = beta; p.g = g;
    p.state = state; p.o = o; p.N = N; p.H = H;
    cudaError_t e = gdn::launch_decode_step(p, Dk, Dv, gate_kind, dtype == GDN_BF16,
                                            reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    g_launches.fetch_add(1);
    return GDN_OK;
}

gdn_status gdn_read_device_status(gdn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, gdn_device_status_word, sizeof(word)) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (word) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(gdn_device_status_word, &zero, sizeof(zero)) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return (word & gdn::kStatusTimeout) ? GDN_ERR_TIMEOUT : GDN_OK;
}

}  // extern "C"
