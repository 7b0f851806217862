// osdn_precondition.cu -- phase 1 of the preconditioned delta rule: the O(d_k)
// scan over the key stream that yields the write keys kw_t = d_t (.) k_t.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", sec. 2.1 (right-preconditioning the gradient step by
// D_t = diag(d_t) is writing along kw_t = d_t (.) k_t), sec. 2.2 (d_t follows
// online gradient descent on the closed-form surrogate
// h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1) / (2 |k_t|^2), which depends on the
// key and beta only), sec. 2.3 (a retention gate r_t scales d before the
// step).  Per (batch, head), token by token:
//     s = <d, k_t^2>,  n = |k_t|^2
//     kw_t = d (.) k_t
//     d   <- r_t d + eta beta_t (1 - beta_t s) k_t^2 / n      (d unchanged if n = 0)
// The scan is sequential in t and independent across (batch, head).  Four
// lanes share one head (each holds a quarter of d in registers), so the two
// dot products of a token need two butterfly shuffles; a warp runs eight
// heads.  The next token's key is loaded while the current one is processed.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int OSDN_THREADS = 128;   // 32 heads per block, 4 lanes each

template <typename Tin, int DK>
__global__ void __launch_bounds__(OSDN_THREADS)
osdn_precondition_kernel(const OsdnParams p) {
    constexpr int PL = DK / 4;                     // dimensions per lane
    const int tid = threadIdx.x;
    const int sub = tid & 3;
    const long long bh = (long long)blockIdx.x * (OSDN_THREADS / 4) + (tid >> 2);
    const bool active = bh < (long long)p.B * p.H;
    const int b = active ? (int)(bh / p.H) : 0, h = active ? (int)(bh % p.H) : 0;
    const Tin* kp = static_cast<const Tin*>(p.k);
    const Tin* bp = static_cast<const Tin*>(p.beta);
    const Tin* rp = static_cast<const Tin*>(p.r);
    Tin* kwp = static_cast<Tin*>(p.kw);
    const unsigned mask = 0xffffffffu;   // every lane runs every token (T is uniform)

    float d[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) d[i] = (active && p.d0) ? p.d0[bh * DK + sub * PL + i] : 1.f;

    auto tok = [&](int t) { return ((long long)b * p.T + t) * p.H + h; };
    // a lane's quarter of a key row: PL elements, 16-byte aligned (rows are
    // DK elements and the base is 16-byte aligned)
    constexpr int NV = PL * (int)sizeof(Tin) / 16;
    float kc[PL], kn[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) kc[i] = kn[i] = 0.f;
    auto load_k = [&](int t, float (&dst)[PL]) {
        const uint4* src = reinterpret_cast<const uint4*>(kp + tok(t) * DK + sub * PL);
        uint4 raw[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) raw[j] = src[j];
        const Tin* e = reinterpret_cast<const Tin*>(raw);
#pragma unroll
        for (int i = 0; i < PL; ++i) dst[i] = to_f32(e[i]);
    };
    if (active && p.T > 0) load_k(0, kc);
#pragma unroll 1
    for (int t = 0; t < p.T; ++t) {
        float bt = 0.f, rt = 1.f;
        if (active) {
            if (t + 1 < p.T) load_k(t + 1, kn);
            bt = to_f32(bp[tok(t)]);
            if (rp) rt = to_f32(rp[tok(t)]);
        }
        float s = 0.f, n = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const float u = kc[i] * kc[i];
            s = fmaf(d[i], u, s);
            n += u;
        }
        s += __shfl_xor_sync(mask, s, 1);
        n += __shfl_xor_sync(mask, n, 1);
        s += __shfl_xor_sync(mask, s, 2);
        n += __shfl_xor_sync(mask, n, 2);
        if (active) {
            uint4 raw[NV];
            Tin* e = reinterpret_cast<Tin*>(raw);
#pragma unroll
            for (int i = 0; i < PL; ++i) e[i] = from_f32<Tin>(d[i] * kc[i]);
            uint4* dst = reinterpret_cast<uint4*>(kwp + tok(t) * DK + sub * PL);
#pragma unroll
            for (int j = 0; j < NV; ++j) dst[j] = raw[j];
        }
        const float e = n > 0.f ? p.eta * bt * (1.f - bt * s) / n : 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) d[i] = fmaf(rt, d[i], e * (kc[i] * kc[i]));
#pragma unroll
        for (int i = 0; i < PL; ++i) kc[i] = kn[i];
    }
    if (active && p.d_out) {
#pragma unroll
        for (int i = 0; i < PL; ++i) p.d_out[bh * DK + sub * PL + i] = d[i];
    }
}

template <typename Tin>
cudaError_t launch_dk(const OsdnParams& p, int Dk, cudaStream_t s) {
    const long long nbh = (long long)p.B * p.H;
    const unsigned grid = (unsigned)((nbh + OSDN_THREADS / 4 - 1) / (OSDN_THREADS / 4));
    if (Dk == 64) return launch_on(osdn_precondition_kernel<Tin, 64>, dim3(grid), dim3(OSDN_THREADS), 0, s, p);
    return launch_on(osdn_precondition_kernel<Tin, 128>, dim3(grid), dim3(OSDN_THREADS), 0, s, p);
}

}  // namespace

cudaError_t launch_osdn_precondition(const OsdnParams& p, int Dk, bool bf16, cudaStream_t s) {
    return bf16 ? launch_dk<__nv_bfloat16>(p, Dk, s) : launch_dk<float>(p, Dk, s);
}

}  // namespace gdn
