// decode_step.cu -- one recurrent gated delta-rule step per (sequence, head).
//
// The constant-size-state decode of the linear layers ("Moonshot AI's New
// Attention Architecture: Key Innovations Explained", sec. 1) for the operator
// of sec. 2 of that page, in M = S^T form (state [Dk][Dv] fp32, row-major):
//     M' = Diag(a) M,  x = M'^T k,  r = beta (v - x),
//     M <- M' + k r^T,  o = M'^T q + r (k . q)
// The step is bound by HBM: the 64 KB state of a d = 128 head is read once and
// written once, everything else is ~1 KB.  One CTA of 8 warps owns one
// (sequence, head); warp w holds rows [w*Dk/8, (w+1)*Dk/8) of M in registers,
// lane l holds columns [l*Dv/32, (l+1)*Dv/32) of each row, so every warp-wide
// load/store is one contiguous 512 B (Dv = 128) row segment.  All state loads
// are issued before the first barrier; x and M'^T q are reduced across warps
// through shared memory; the update is written back from the same registers.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int NW = 8;
constexpr int NT = NW * 32;

template <int VPL> struct Vec;
template <> struct Vec<4> {
    static __device__ __forceinline__ void load(const float* p, float* r) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        r[0] = t.x; r[1] = t.y; r[2] = t.z; r[3] = t.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* r) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(r[0], r[1], r[2], r[3]));
    }
};
template <> struct Vec<2> {
    static __device__ __forceinline__ void load(const float* p, float* r) {
        const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
        r[0] = t.x; r[1] = t.y;
    }
    static __device__ __forceinline__ void store(float* p, const float* r) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(r[0], r[1]));
    }
};

template <typename Tin, int DK, int DV, int GATE>
__global__ void __launch_bounds__(NT) decode_step_kernel(DecodeParams p) {
    constexpr int ROWS = DK / NW;
    constexpr int VPL = DV / 32;
    __shared__ float ks[DK], qs[DK], as[DK];
    __shared__ float sx[NW][DV], sy[NW][DV], skq[NW];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t nh = blockIdx.x;
    float* M = p.state + nh * (size_t)(DK * DV);
    const Tin* q = static_cast<const Tin*>(p.q) + nh * DK;
    const Tin* k = static_cast<const Tin*>(p.k) + nh * DK;
    const Tin* v = static_cast<const Tin*>(p.v) + nh * DV;
    const int col0 = lane * VPL;
    const int row0 = warp * ROWS;

    float m[ROWS][VPL];
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) Vec<VPL>::load(M + (size_t)(row0 + rr) * DV + col0, m[rr]);

    for (int i = tid; i < DK; i += NT) {
        ks[i] = to_f32(k[i]);
        qs[i] = to_f32(q[i]);
        if constexpr (GATE == kGatePerDim)
            as[i] = expf(to_f32(static_cast<const Tin*>(p.g)[nh * DK + i]));
    }
    float vv[VPL];
#pragma unroll
    for (int c = 0; c < VPL; ++c) vv[c] = to_f32(v[col0 + c]);
    const float bt = to_f32(static_cast<const Tin*>(p.beta)[nh]);
    float a_scalar = 1.f;
    if constexpr (GATE == kGateScalar) a_scalar = expf(to_f32(static_cast<const Tin*>(p.g)[nh]));
    __syncthreads();

    float px[VPL], py[VPL];
#pragma unroll
    for (int c = 0; c < VPL; ++c) { px[c] = 0.f; py[c] = 0.f; }
    float kq = 0.f;
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) {
        const int i = row0 + rr;
        const float ki = ks[i], qi = qs[i];
        kq = fmaf(ki, qi, kq);
        float a = a_scalar;
        if constexpr (GATE == kGatePerDim) a = as[i];
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
            if constexpr (GATE != kGateNone) m[rr][c] *= a;
            px[c] = fmaf(m[rr][c], ki, px[c]);
            py[c] = fmaf(m[rr][c], qi, py[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < VPL; ++c) { sx[warp][col0 + c] = px[c]; sy[warp][col0 + c] = py[c]; }
    if (lane == 0) skq[warp] = kq;
    __syncthreads();

    float r[VPL];
    float kq_all = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) kq_all += skq[w];
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
        float x = 0.f, y = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) { x += sx[w][col0 + c]; y += sy[w][col0 + c]; }
        r[c] = bt * (vv[c] - x);
        if (warp == 0)
            static_cast<Tin*>(p.o)[nh * DV + col0 + c] = from_f32<Tin>(fmaf(r[c], kq_all, y));
    }
#pragma unroll
    for (int rr = 0; rr < ROWS; ++rr) {
        const float ki = ks[row0 + rr];
#pragma unroll
        for (int c = 0; c < VPL; ++c) m[rr][c] = fmaf(ki, r[c], m[rr][c]);
        Vec<VPL>::store(M + (size_t)(row0 + rr) * DV + col0, m[rr]);
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_gate(const DecodeParams& p, int gate, cudaStream_t s) {
    const unsigned grid = (unsigned)((size_t)p.N * p.H);
    auto kern = gate == kGateNone     ? decode_step_kernel<Tin, DK, DV, kGateNone>
                : gate == kGateScalar ? decode_step_kernel<Tin, DK, DV, kGateScalar>
                                      : decode_step_kernel<Tin, DK, DV, kGatePerDim>;
    return launch_on(kern, dim3(grid), dim3(NT), 0, s, p);
}

template <typename Tin>
cudaError_t launch_dims(const DecodeParams& p, int Dk, int Dv, int gate, cudaStream_t s) {
    if (Dk == 128 && Dv == 128) return launch_gate<Tin, 128, 128>(p, gate, s);
    if (Dk == 128 && Dv == 64) return launch_gate<Tin, 128, 64>(p, gate, s);
    if (Dk == 64 && Dv == 128) return launch_gate<Tin, 64, 128>(p, gate, s);
    return launch_gate<Tin, 64, 64>(p, gate, s);
}

}  // namespace

cudaError_t launch_decode_step(const DecodeParams& p, int Dk, int Dv, int gate, bool bf16,
                               cudaStream_t s) {
    return bf16 ? launch_dims<__nv_bfloat16>(p, Dk, Dv, gate, s)
                : launch_dims<float>(p, Dk, Dv, gate, s);
}

}  // namespace gdn
