// chunk_fwd_simt.cu -- chunkwise gated delta rule on CUDA cores, fp32 math.
//
// The fp32 path of gdn_chunk_fwd.  fp32 inputs need fp32 accumulation end to
// end (tensor-core tf32 keeps a 10-bit mantissa), so every product here is an
// fp32 FMA.  One CTA owns one (batch, head, 32-column block of d_v): the d_v
// columns of the state evolve independently, so the split is exact and needs
// no communication between CTAs.
//
// Per chunk of C = 64 tokens (the chunkwise state recurrence and output of
// "Moonshot AI's New Attention Architecture: Key Innovations Explained",
// sec. 3; the UT/WY transform of "OSDN: Improving Delta Rule with Provable
// Online Preconditioning in Linear Attention", sec. 2.1), h = entering state:
//   G_r   = sum_{i<=r} g_i                 log-domain cumulative decay
//   A_ri  = beta_r sum_d k_rd k_id e^(G_rd - G_id)   (i < r)
//   P_ri  = sum_d q_rd k_id e^(G_rd - G_id)          (i <= r)
//   T     = (I + A)^-1                      forward substitution
//   E     = diag(beta) (V - K_bar h)        K_bar = e^G * K
//   D     = T E                             (= U - W h with U, W the WY factors)
//   O     = Q_bar h + P D                   Q_bar = e^G * Q
//   h'    = e^(G_C) * h + K_tilde^T D       K_tilde_i = e^(G_C - G_i) * k_i
// Every exponent above is <= 0 for the entries used, so nothing overflows.
// Rows past the end of the sequence are zero with beta = 0 and g = 0, which
// leaves the state untouched.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int BV = 32;
constexpr int NT = 256;

template <int DK, int GATE>
struct SimtSmem {
    static constexpr int LD = DK + 1;           // padded row of a [C][DK] tile
    static constexpr int kK = 0;                              // K raw
    static constexpr int kQ = kK + C * LD;                    // Q, then Q_bar
    static constexpr int kX = kQ + C * LD;                    // K_bar, then K_tilde (per-dim)
    static constexpr int kG = kX + (GATE == kGatePerDim ? C * LD : 0);   // G [C][LD] or [C]
    static constexpr int kV = kG + (GATE == kGatePerDim ? C * LD : C);   // V, then E
    static constexpr int kD = kV + C * (BV + 1);              // D
    static constexpr int kA = kD + C * (BV + 1);              // A
    static constexpr int kP = kA + C * (C + 1);               // P
    static constexpr int kT = kP + C * (C + 1);               // T
    static constexpr int kH = kT + C * (C + 1);               // state block [DK][BV+1]
    static constexpr int kBeta = kH + DK * (BV + 1);
    static constexpr int kGam = kBeta + C;                    // e^G_r (scalar gate)
    static constexpr int kFt = kGam + C;                      // e^(G_C - G_r) (scalar gate)
    static constexpr int kTotal = kFt + C;
    static constexpr size_t bytes = sizeof(float) * (size_t)kTotal;
};

template <typename Tin, int DK, int GATE>
__global__ void __launch_bounds__(NT) chunk_fwd_simt_kernel(ChunkParams p) {
    using L = SimtSmem<DK, GATE>;
    constexpr int LD = L::LD;
    extern __shared__ float sm[];
    float* Ks = sm + L::kK;
    float* Qs = sm + L::kQ;
    float* Xs = sm + L::kX;
    float* Gs = sm + L::kG;
    float* Vs = sm + L::kV;
    float* Ds = sm + L::kD;
    float* As = sm + L::kA;
    float* Ps = sm + L::kP;
    float* Ts = sm + L::kT;
    float* Hs = sm + L::kH;
    float* betas = sm + L::kBeta;
    float* Gam = sm + L::kGam;
    float* Ft = sm + L::kFt;

    const int tid = threadIdx.x;
    const int H = p.H, T = p.T, Dv = p.Dv;
    const int nvb = Dv / BV;
    const int v0 = (int)(blockIdx.x % nvb) * BV;
    const int h = (int)((blockIdx.x / nvb) % H);
    const int b = (int)(blockIdx.x / nvb / H);
    const Tin* q = static_cast<const Tin*>(p.q);
    const Tin* k = static_cast<const Tin*>(p.k);
    const Tin* v = static_cast<const Tin*>(p.v);
    const Tin* beta = static_cast<const Tin*>(p.beta);
    const Tin* g = static_cast<const Tin*>(p.g);
    Tin* o = static_cast<Tin*>(p.o);
    const size_t state_off = ((size_t)b * H + h) * DK * Dv;

    for (int idx = tid; idx < DK * BV; idx += NT) {
        const int d = idx / BV, c = idx % BV;
        Hs[d * (BV + 1) + c] = p.s0 ? p.s0[state_off + (size_t)d * Dv + v0 + c] : 0.f;
    }

    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        __syncthreads();
        // ---- load the chunk (rows >= n are zero, beta = 0, g = 0); every load
        // of a thread is issued before the first is stored, so the chunk costs
        // one memory latency rather than one per element
        {
            constexpr int PK = C * DK / NT, PV = C * BV / NT;
            static_assert(C * DK % NT == 0 && C * BV % NT == 0, "whole rounds");
            float kv[PK], qv[PK], gv[GATE == kGatePerDim ? PK : 1], vv[PV];
#pragma unroll
            for (int m = 0; m < PK; ++m) {
                const int idx = tid + m * NT, r = idx / DK, d = idx % DK;
                const size_t tok = ((size_t)b * T + t0 + r) * H + h;
                const bool ok = r < n;
                kv[m] = ok ? to_f32(k[tok * DK + d]) : 0.f;
                qv[m] = ok ? to_f32(q[tok * DK + d]) : 0.f;
                if constexpr (GATE == kGatePerDim) gv[m] = ok ? to_f32(g[tok * DK + d]) : 0.f;
            }
#pragma unroll
            for (int m = 0; m < PV; ++m) {
                const int idx = tid + m * NT, r = idx / BV, c = idx % BV;
                const size_t tok = ((size_t)b * T + t0 + r) * H + h;
                vv[m] = r < n ? to_f32(v[tok * Dv + v0 + c]) : 0.f;
            }
#pragma unroll
            for (int m = 0; m < PK; ++m) {
                const int idx = tid + m * NT, r = idx / DK, d = idx % DK;
                Ks[r * LD + d] = kv[m];
                Qs[r * LD + d] = qv[m];
                if constexpr (GATE == kGatePerDim) Gs[r * LD + d] = gv[m];
            }
#pragma unroll
            for (int m = 0; m < PV; ++m) {
                const int idx = tid + m * NT, r = idx / BV, c = idx % BV;
                Vs[r * (BV + 1) + c] = vv[m];
            }
        }
        if (tid < C) {
            const size_t tok = ((size_t)b * T + t0 + tid) * H + h;
            betas[tid] = tid < n ? to_f32(beta[tok]) : 0.f;
            if constexpr (GATE == kGateScalar) Gs[tid] = tid < n ? to_f32(g[tok]) : 0.f;
        }
        __syncthreads();
        // ---- log-domain cumulative decay within the chunk
        if constexpr (GATE == kGateScalar) {
            if (tid == 0) {
                float acc = 0.f;
                for (int r = 0; r < C; ++r) { acc += Gs[r]; Gs[r] = acc; }
            }
            __syncthreads();
            if (tid < C) {
                Gam[tid] = expf(Gs[tid]);
                Ft[tid] = expf(Gs[C - 1] - Gs[tid]);
            }
        } else if constexpr (GATE == kGatePerDim) {
            if (tid < DK) {
                float acc = 0.f;
                for (int r = 0; r < C; ++r) { acc += Gs[r * LD + tid]; Gs[r * LD + tid] = acc; }
            }
        } else {
            if (tid < C) { Gam[tid] = 1.f; Ft[tid] = 1.f; }
        }
        __syncthreads();
        // ---- intra-chunk system A and causal scores P (raw K, Q)
        for (int idx = tid; idx < C * C; idx += NT) {
            const int r = idx / C, i = idx % C;
            float a = 0.f, s = 0.f;
            if (i <= r) {
                if constexpr (GATE == kGatePerDim) {
                    for (int d = 0; d < DK; ++d) {
                        const float e = expf(Gs[r * LD + d] - Gs[i * LD + d]);
                        const float ki = Ks[i * LD + d] * e;
                        a = fmaf(Ks[r * LD + d], ki, a);
                        s = fmaf(Qs[r * LD + d], ki, s);
                    }
                } else {
                    for (int d = 0; d < DK; ++d) {
                        a = fmaf(Ks[r * LD + d], Ks[i * LD + d], a);
                        s = fmaf(Qs[r * LD + d], Ks[i * LD + d], s);
                    }
                    if constexpr (GATE == kGateScalar) {
                        const float e = expf(Gs[r] - Gs[i]);
                        a *= e;
                        s *= e;
                    }
                }
                a = (i < r) ? betas[r] * a : 0.f;
            }
            As[r * (C + 1) + i] = a;
            Ps[r * (C + 1) + i] = s;
        }
        if constexpr (GATE == kGatePerDim) {
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += NT) {
                const int r = idx / DK, d = idx % DK;
                const float e = expf(Gs[r * LD + d]);
                Xs[r * LD + d] = Ks[r * LD + d] * e;   // K_bar
                Qs[r * LD + d] = Qs[r * LD + d] * e;   // Q_bar
            }
        }
        __syncthreads();
        // ---- E = diag(beta) (V - K_bar h)
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int r = idx / BV, c = idx % BV;
            float x = 0.f;
            if constexpr (GATE == kGatePerDim) {
                for (int d = 0; d < DK; ++d) x = fmaf(Xs[r * LD + d], Hs[d * (BV + 1) + c], x);
            } else {
                for (int d = 0; d < DK; ++d) x = fmaf(Ks[r * LD + d], Hs[d * (BV + 1) + c], x);
                x *= Gam[r];
            }
            Vs[r * (BV + 1) + c] = betas[r] * (Vs[r * (BV + 1) + c] - x);
        }
        // ---- T = (I + A)^-1 by forward substitution: 4 threads per column j
        {
            const int j = tid >> 2, s = tid & 3;
            for (int r = 0; r < C; ++r) {
                float part = 0.f;
                for (int i = j + s; i < r; i += 4) part = fmaf(As[r * (C + 1) + i], Ts[i * (C + 1) + j], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                if (s == 0) Ts[r * (C + 1) + j] = (r == j) ? 1.f : (r > j ? -part : 0.f);
                __syncwarp();
            }
        }
        __syncthreads();
        // ---- D = T E
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int r = idx / BV, c = idx % BV;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Ts[r * (C + 1) + i], Vs[i * (BV + 1) + c], acc);
            Ds[r * (BV + 1) + c] = acc;
        }
        __syncthreads();
        // ---- O = Q_bar h + P D ; K_tilde (per-dim) into Xs
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int r = idx / BV, c = idx % BV;
            if (r >= n) continue;
            float acc = 0.f;
            for (int d = 0; d < DK; ++d) acc = fmaf(Qs[r * LD + d], Hs[d * (BV + 1) + c], acc);
            if constexpr (GATE != kGatePerDim) acc *= Gam[r];
            for (int i = 0; i <= r; ++i) acc = fmaf(Ps[r * (C + 1) + i], Ds[i * (BV + 1) + c], acc);
            const size_t tok = ((size_t)b * T + t0 + r) * H + h;
            o[tok * Dv + v0 + c] = from_f32<Tin>(acc);
        }
        if constexpr (GATE == kGatePerDim) {
            for (int idx = tid; idx < C * DK; idx += NT) {
                const int r = idx / DK, d = idx % DK;
                Xs[r * LD + d] = Ks[r * LD + d] * expf(Gs[(C - 1) * LD + d] - Gs[r * LD + d]);
            }
        }
        __syncthreads();
        // ---- h' = e^(G_C) h + K_tilde^T D
        for (int idx = tid; idx < DK * BV; idx += NT) {
            const int d = idx / BV, c = idx % BV;
            float acc;
            if constexpr (GATE == kGatePerDim) {
                acc = expf(Gs[(C - 1) * LD + d]) * Hs[d * (BV + 1) + c];
                for (int i = 0; i < C; ++i) acc = fmaf(Xs[i * LD + d], Ds[i * (BV + 1) + c], acc);
            } else {
                acc = Gam[C - 1] * Hs[d * (BV + 1) + c];
                for (int i = 0; i < C; ++i)
                    acc = fmaf(Ks[i * LD + d] * Ft[i], Ds[i * (BV + 1) + c], acc);
            }
            Hs[d * (BV + 1) + c] = acc;
        }
    }
    __syncthreads();
    if (p.s_out) {
        for (int idx = tid; idx < DK * BV; idx += NT) {
            const int d = idx / BV, c = idx % BV;
            p.s_out[state_off + (size_t)d * Dv + v0 + c] = Hs[d * (BV + 1) + c];
        }
    }
}

template <typename Tin, int DK, int GATE>
cudaError_t launch_typed(const ChunkParams& p, cudaStream_t s) {
    using L = SimtSmem<DK, GATE>;
    auto kern = chunk_fwd_simt_kernel<Tin, DK, GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::bytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)(p.Dv / BV) * p.H * p.B);
    return launch_on(kern, dim3(grid), dim3(NT), L::bytes, s, p);
}

template <typename Tin>
cudaError_t launch_dk(const ChunkParams& p, int gate, cudaStream_t s) {
    if (p.Dk == 64) {
        if (gate == kGateNone) return launch_typed<Tin, 64, kGateNone>(p, s);
        if (gate == kGateScalar) return launch_typed<Tin, 64, kGateScalar>(p, s);
        return launch_typed<Tin, 64, kGatePerDim>(p, s);
    }
    if (gate == kGateNone) return launch_typed<Tin, 128, kGateNone>(p, s);
    if (gate == kGateScalar) return launch_typed<Tin, 128, kGateScalar>(p, s);
    return launch_typed<Tin, 128, kGatePerDim>(p, s);
}

}  // namespace

cudaError_t launch_chunk_fwd_simt(const ChunkParams& p, int gate, bool bf16, cudaStream_t s) {
    return bf16 ? launch_dk<__nv_bfloat16>(p, gate, s) : launch_dk<float>(p, gate, s);
}

}  // namespace gdn
