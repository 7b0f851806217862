// common.cuh -- small device helpers shared by the libgdn kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

enum Gate : int { kGateNone = 0, kGateScalar = 1, kGatePerDim = 2 };

// Bits of the library's device status word (set by kernels that give up a
// bounded wait; read and cleared by gdn_read_device_status).
enum StatusBits : unsigned { kStatusTimeout = 1u };

struct ChunkParams {
    const void* q;
    const void* k;
    const void* v;
    const void* beta;
    const void* g;
    const void* kw;    // write key [B, T, H, Dk] (preconditioned delta rule), or null (= k)
    const float* s0;   // may be null
    void* o;
    float* s_out;      // may be null
    int B, T, H, Dk, Dv;
    unsigned* status;  // device status word
    // tensor-core path: workspace and the wave of chunks one launch pair covers
    uint8_t* ws;       // per-chunk prep images, [B*H][cw] x WS_CHUNK bytes
    int cw;            // chunk slots per (batch, head) in the workspace
    int chunk0;        // first chunk of this wave
    int nchunks;       // chunks in this wave
    int ws_chunk;      // bytes of one chunk's workspace image
    unsigned* counter; // this wave's item counter (persistent prep CTAs take items from it)
    // segment-parallel state pass (seg_mode 0: one chain CTA per (batch, head))
    int seg_mode;      // 1: offsets and transitions of every segment; 3: outputs of every segment
    int nseg, seg_len; // segments per (batch, head) in this wave, chunks per segment
    float* seg_h;      // [B*H][nseg][Dk][Dv] entering state of each segment (j >= 1)
    // backward support: the entering state of every chunk, fp32 [B*H][nchunks][Dk][Dv]
    float* h_all;      // null: not kept
    int nc_total;      // chunks per (batch, head) of the whole sequence
};

// Phase 1 of the preconditioned delta rule (write keys kw = d (.) k).
struct OsdnParams {
    const void* k;       // [B, T, H, Dk]
    const void* beta;    // [B, T, H]
    const void* r;       // [B, T, H] retention gate, or null (r = 1)
    void* kw;            // [B, T, H, Dk] write keys (output)
    const float* d0;     // [B, H, Dk] initial preconditioner, or null (ones)
    float* d_out;        // [B, H, Dk] final preconditioner (output), or null
    float eta;           // step size of the preconditioner's gradient descent
    int B, T, H;
};

// Backward of the chunk forward (scalar gate or none, bf16 inputs, d = 128).
struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const void* beta;
    const void* g;       // [B, T, H] (scalar gate) or null
    const void* dO;      // [B, T, H, Dv] upstream gradient of o, bf16
    const float* dS;     // [B, H, Dk, Dv] upstream gradient of the final state, or null
    float* dq;           // [B, T, H, Dk] fp32
    float* dk;           // [B, T, H, Dk] fp32
    float* dv;           // [B, T, H, Dv] fp32
    float* dbeta;        // [B, T, H] fp32
    float* dg;           // [B, T, H] fp32 (scalar gate) or null
    float* dS0;          // [B, H, Dk, Dv] fp32 or null
    const uint8_t* images;   // the forward's step images, [B*H][NC]
    float* h_all;        // entering state of every chunk
    float* dh_all;       // adjoint of every chunk's leaving state
    unsigned* status;    // device status word (a bounded wait that gave up)
    int B, T, H;
};

struct DecodeParams {
    const void* q;
    const void* k;
    const void* v;
    const void* beta;
    const void* g;
    float* state;
    void* o;
    int N, H;
};

// Launches `kern` on `s` and returns that launch's own error (never one left
// over from an earlier call, which cudaGetLastError after a <<<>>> launch
// would report).
template <typename... Params, typename... Args>
inline cudaError_t launch_on(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace gdn

// Launchers implemented in the kernel translation units.
namespace gdn {
cudaError_t launch_chunk_fwd_simt(const ChunkParams& p, int gate, bool bf16, cudaStream_t s);
bool chunk_fwd_tc_supported(int Dk, int Dv, int gate);
// Workspace for the longest waves the forward uses / the least it runs with.
size_t chunk_fwd_tc_workspace_bytes(int B, int T, int H, int gate);
size_t chunk_fwd_tc_workspace_min_bytes(int B, int T, int H, int gate);
// Waves, chunks per wave and segments per wave of a forward with ws_bytes.
void chunk_fwd_tc_plan(int B, int T, int H, int gate, size_t ws_bytes, int* waves,
                       int* chunks_per_wave, int* segments);
// Enqueues the tensor-core forward with a workspace of ws_bytes (at least the
// minimum; waves as long as it allows); *launches receives the number of
// kernels.
cudaError_t launch_chunk_fwd_tc(const ChunkParams& p, int gate, size_t ws_bytes, cudaStream_t s,
                                int* launches);
cudaError_t launch_decode_step(const DecodeParams& p, int Dk, int Dv, int gate, bool bf16,
                               cudaStream_t s);
// Phase 1 of the preconditioned delta rule in blocks of 64 tokens (three
// launches); ws holds osdn_precondition_workspace_bytes(B, T, H, Dk).
size_t osdn_precondition_workspace_bytes(int B, int T, int H, int Dk);
cudaError_t launch_osdn_precondition(const OsdnParams& p, int Dk, bool bf16, uint8_t* ws,
                                     cudaStream_t s, int* launches);
// The forward in one wave, keeping every chunk's step image in ws (at offset 0,
// [B*H][NC] images) and every chunk's entering state in h_all.  ws_bytes >=
// chunk_fwd_tc_capture_bytes.
size_t chunk_fwd_tc_capture_bytes(int B, int T, int H);
cudaError_t launch_chunk_fwd_tc_capture(const ChunkParams& p, int gate, size_t ws_bytes,
                                        float* h_all, cudaStream_t s, int* launches);
size_t chunk_bwd_workspace_bytes(int B, int T, int H);
cudaError_t launch_chunk_bwd(const ChunkParams& pf, const BwdParams& pb, int gate, uint8_t* ws,
                             size_t ws_bytes, cudaStream_t s, int* launches);
// Image layout facts the backward reads (bytes): the [Phi ; Qp] operand and gamma.
constexpr uint32_t kImgBytes = 90624, kImgPQ = 0, kImgPQBlock = 24576, kImgGam = 90112;
}  // namespace gdn
