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
//     s_t = <d_t, u_t>,  u_t = k_t (.) k_t,  n_t = |k_t|^2
//     kw_t = d_t (.) k_t
//     d_{t+1} = r_t d_t + e_t u_t,   e_t = a_t - c_t s_t,
//     a_t = eta beta_t / n_t,  c_t = eta beta_t^2 / n_t     (a_t = c_t = 0 if n_t = 0)
// The step e_t is affine in s_t, and s_t is linear in the entering d and the
// earlier steps, so a block of L tokens entering with d_0 solves a
// lower-triangular system (plain algebra on the lines above, not printed on
// the page):
//     d_t = R_t d_0 + sum_{j<t} R_{j->t} e_j u_j,  R_t = prod_{i<t} r_i,
//           R_{j->t} = prod_{j<i<t} r_i
//     (I + Lm) e = a - c (.) R (.) p,   p_t = <d_0, u_t>,
//           Lm_tj = c_t R_{j->t} <u_j, u_t>  (j < t)
//     d_L = R_L d_0 + sum_j R_{j->L} e_j u_j.
// Only p (and so e and d_L) depends on d_0.  Three launches:
//   osdn_block_kernel  every block at once: u, n, a, c, the Gram matrix of the
//                      u, Lm and T = (I + Lm)^-1 (forward substitution);
//   osdn_chain_kernel  per (batch, head), blocks in order: p = U d_0,
//                      e = T (a - c R p), d_L; stores each block's d_0 and e;
//   osdn_write_kernel  every block at once: kw_t = d_t (.) k_t from d_0 and e.
// All arithmetic in fp32.
#include "common.cuh"

namespace gdn {
namespace {

constexpr int L = 64;                  // tokens a block
constexpr int OB_THREADS = 256;
constexpr int LDL = L + 1;             // fp32 row stride of [L][L] matrices

// Workspace per block (bytes): T [L][L] fp32, then the vectors a, cR = c R,
// rho_j = R_{j->L}, misc (misc[0] = R_L), e, and d_0 [Dk].
constexpr size_t WS_T = (size_t)L * L * 4;
constexpr size_t WS_VEC = 5 * L * 4;
__host__ __device__ inline size_t ws_block_bytes(int Dk) { return WS_T + WS_VEC + (size_t)Dk * 4; }

struct BlockWs {
    float* T;
    float* a;
    float* cR;
    float* rho;
    float* misc;
    float* e;
    float* d0;
};
__device__ inline BlockWs block_ws(uint8_t* ws, long long q, int Dk) {
    uint8_t* base = ws + (size_t)q * ws_block_bytes(Dk);
    BlockWs w;
    w.T = reinterpret_cast<float*>(base);
    float* v = reinterpret_cast<float*>(base + WS_T);
    w.a = v;
    w.cR = v + L;
    w.rho = v + 2 * L;
    w.misc = v + 3 * L;
    w.e = v + 4 * L;
    w.d0 = v + 5 * L;
    return w;
}

// u = k (.) k of block c of (b, h) into us [L][Dk + 1] (rows past T zero):
// 16-byte loads, all of a thread's issued before the first is used
template <typename Tin, int DK, int NT>
__device__ inline void load_u(const OsdnParams& p, int b, int h, int c, float* us, int tid) {
    constexpr int EPV = 16 / (int)sizeof(Tin);        // elements a 16-byte load
    constexpr int VPR = DK / EPV;                     // loads a row
    constexpr int PER = L * VPR / NT;                 // loads a thread
    static_assert(L * VPR % NT == 0, "whole loads a thread");
    const Tin* kp = static_cast<const Tin*>(p.k);
    uint4 raw[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int idx = tid + NT * m, t = idx / VPR, j = idx % VPR, tg = c * L + t;
        raw[m] = make_uint4(0u, 0u, 0u, 0u);
        if (tg < p.T)
            raw[m] = *reinterpret_cast<const uint4*>(kp + (((size_t)b * p.T + tg) * p.H + h) * DK + j * EPV);
    }
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int idx = tid + NT * m, t = idx / VPR, j = idx % VPR;
        const Tin* e = reinterpret_cast<const Tin*>(&raw[m]);
#pragma unroll
        for (int q = 0; q < EPV; ++q) {
            const float x = to_f32(e[q]);
            us[t * (DK + 1) + j * EPV + q] = x * x;
        }
    }
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(OB_THREADS)
osdn_block_kernel(const OsdnParams p, uint8_t* ws) {
    extern __shared__ float smf[];
    float* us = smf;                          // u [L][DK + 1]
    float* Lm = us + L * (DK + 1);            // Lm [L][LDL]
    float* Rm = Lm + L * LDL;                 // R_{j->t} [L][LDL]
    float* sv = Rm + L * LDL;                 // a, c, r [L] each, then a [32][33] scratch
    float* sa = sv, *sc = sv + L, *sr = sv + 2 * L;
    const int NB = (p.T + L - 1) / L;
    const long long q = blockIdx.x;
    const int bh = (int)(q / NB), c = (int)(q % NB), b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const BlockWs w = block_ws(ws, q, DK);
    load_u<Tin, DK, OB_THREADS>(p, b, h, c, us, tid);
    if (tid < L) {
        const int tg = c * L + tid;
        float bt = 0.f, rt = 1.f;
        if (tg < p.T) {
            const size_t tk = ((size_t)b * p.T + tg) * p.H + h;
            bt = to_f32(static_cast<const Tin*>(p.beta)[tk]);
            if (p.r) rt = to_f32(static_cast<const Tin*>(p.r)[tk]);
        }
        sa[tid] = bt;
        sr[tid] = rt;
    }
    __syncthreads();
    // n_t = sum_d u_td (a warp per row), then a_t, c_t
    for (int t = warp; t < L; t += OB_THREADS / 32) {
        float s = 0.f;
        for (int dd = lane; dd < DK; dd += 32) s += us[t * (DK + 1) + dd];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            const float bt = sa[t];
            sa[t] = s > 0.f ? p.eta * bt / s : 0.f;
            sc[t] = s > 0.f ? p.eta * bt * bt / s : 0.f;
        }
    }
    __syncthreads();
    // R_{j->t} row by row from the diagonal (one thread a row t)
    if (tid < L) {
        const int t = tid;
        float rp = 1.f;
        for (int j = t - 1; j >= 0; --j) {
            Rm[t * LDL + j] = rp;
            rp *= sr[j];
        }
    }
    // Gram matrix <u_t, u_j>: thread (tr, tc) holds rows 16 a + tr, columns
    // 16 b + tc (a warp reads one row of u per step for two rows t and 16
    // consecutive rows j: broadcast and conflict-free)
    {
        const int tr = tid >> 4, tc = tid & 15;
        float g[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) g[a][bb] = 0.f;
#pragma unroll 4
        for (int dd = 0; dd < DK; ++dd) {
            float ut[4], uj[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) ut[a] = us[(16 * a + tr) * (DK + 1) + dd];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) uj[bb] = us[(16 * bb + tc) * (DK + 1) + dd];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb <= a; ++bb) g[a][bb] = fmaf(ut[a], uj[bb], g[a][bb]);
        }   // (tiles above the diagonal, bb > a, are never used)
        __syncthreads();   // R_{j->t} is complete
        // Lm_tj = c_t R_{j->t} <u_j, u_t> for j < t
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int t = 16 * a + tr, j = 16 * bb + tc;
                Lm[t * LDL + j] = j < t ? sc[t] * Rm[t * LDL + j] * g[a][bb] : 0.f;
            }
    }
    __syncthreads();
    // T = (I + Lm)^-1 in blocks (R_{j->t} is dead: Ts takes its place):
    // (1) the four 16 x 16 diagonal inverses by substitution, one column a
    // thread; (2) 16 -> 32: T_10 = -D_1 (Lm_10 D_0) for the two 32 x 32
    // diagonal blocks; (3) 32 -> 64 the same with 32 x 32 blocks.  Every sum
    // runs over the lower-triangular parts only.
    float* Ts = Rm;
    if (tid < L) {
        const int o = 16 * (tid >> 4), c = tid & 15;
        float pr[16], x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) pr[r] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            x[i] = (i == c) ? 1.f : (i < c ? 0.f : -pr[i]);
#pragma unroll
            for (int r = i + 1; r < 16; ++r) pr[r] = fmaf(Lm[(o + r) * LDL + o + i], x[i], pr[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Ts[(o + r) * LDL + o + c] = x[r];
    }
    __syncthreads();
    float* Xs = sv + 3 * L;   // scratch [32][33]
    {   // (2): pair pp of diagonal blocks (2 pp + 1, 2 pp); thread: row r, columns c0, c0 + 1
        const int pp = tid >> 7, idx = tid & 127, r = idx >> 3, c0 = 2 * (idx & 7);
        const int ri = 32 * pp + 16, cj = 32 * pp;
        float x0 = 0.f, x1 = 0.f;
        for (int i = c0; i < 16; ++i) {
            const float lm = Lm[(ri + r) * LDL + cj + i];
            x0 = fmaf(lm, Ts[(cj + i) * LDL + cj + c0], x0);
            if (i > c0) x1 = fmaf(lm, Ts[(cj + i) * LDL + cj + c0 + 1], x1);
        }
        Xs[(16 * pp + r) * 33 + c0] = x0;
        Xs[(16 * pp + r) * 33 + c0 + 1] = x1;
        __syncthreads();
        float t0 = 0.f, t1 = 0.f;
        for (int i = 0; i <= r; ++i) {
            const float d1 = Ts[(ri + r) * LDL + ri + i];
            t0 = fmaf(d1, Xs[(16 * pp + i) * 33 + c0], t0);
            t1 = fmaf(d1, Xs[(16 * pp + i) * 33 + c0 + 1], t1);
        }
        Ts[(ri + r) * LDL + cj + c0] = -t0;
        Ts[(ri + r) * LDL + cj + c0 + 1] = -t1;
    }
    __syncthreads();
    {   // (3): thread: row r of the 32 x 32 block, columns c0 .. c0 + 3
        const int r = tid >> 3, c0 = 4 * (tid & 7);
        float xv[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = c0; i < 32; ++i) {
            const float lm = Lm[(32 + r) * LDL + i];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (i >= c0 + q) xv[q] = fmaf(lm, Ts[i * LDL + c0 + q], xv[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) Xs[r * 33 + c0 + q] = xv[q];
        __syncthreads();
        float tv[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i <= r; ++i) {
            const float t11 = Ts[(32 + r) * LDL + 32 + i];
#pragma unroll
            for (int q = 0; q < 4; ++q) tv[q] = fmaf(t11, Xs[i * 33 + c0 + q], tv[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) Ts[(32 + r) * LDL + c0 + q] = -tv[q];
    }
    __syncthreads();
    for (int idx = tid; idx < L * L; idx += OB_THREADS) {   // lower triangle, zeros above
        const int r = idx >> 6, cc = idx & 63;
        w.T[idx] = cc <= r ? Ts[r * LDL + cc] : 0.f;
    }
    // vectors: R_t = prod_{i<t} r_i, cR_t = c_t R_t, rho_j = prod_{j<i<L} r_i, R_L
    if (tid == 64) {
        float R = 1.f;
        for (int t = 0; t < L; ++t) {
            w.a[t] = sa[t];
            w.cR[t] = sc[t] * R;
            R *= sr[t];
        }
        w.misc[0] = R;
        float rp = 1.f;
        for (int j = L - 1; j >= 0; --j) {
            w.rho[j] = rp;
            rp *= sr[j];
        }
    }
}

// One CTA per (batch, head): the blocks in order, d in shared memory.  The
// next block's keys (raw, rows padded by 16 bytes), its T and its vectors are
// copied in (cp.async) while the current block is worked on; u = k^2 is formed
// where it is used.
__device__ __forceinline__ void cp_async16_zf(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int OC_THREADS = 256;
template <typename Tin>
constexpr int chain_row_stride(int DK) { return DK * (int)sizeof(Tin) + 16; }
template <typename Tin, int DK>
constexpr size_t chain_smem() {
    return 2 * ((size_t)L * chain_row_stride<Tin>(DK) + (size_t)L * L * 4 + 4 * L * 4) +
           (size_t)(DK + 2 * L) * 4;
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(OC_THREADS)
osdn_chain_kernel(const OsdnParams p, uint8_t* ws) {
    constexpr int RB = DK * (int)sizeof(Tin);          // bytes of a key row
    constexpr int RS = chain_row_stride<Tin>(DK);      // its padded stride in shared memory
    constexpr size_t BUF = (size_t)L * RS + (size_t)L * L * 4 + 4 * L * 4;
    extern __shared__ __align__(16) uint8_t smb[];
    float* sd = reinterpret_cast<float*>(smb + 2 * BUF);   // d [DK]
    float* sw = sd + DK;                                    // w [L]
    float* se = sw + L;                                     // e [L]
    const int NB = (p.T + L - 1) / L;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x;
    const uint8_t* kbytes = static_cast<const uint8_t*>(p.k);
    // block c into buffer c & 1: keys, T, then a, cR, rho, misc (contiguous in
    // the workspace)
    auto stage = [&](int c) {
        uint8_t* buf = smb + (c & 1) * BUF;
        for (int idx = tid; idx < L * (RB / 16); idx += OC_THREADS) {
            const int t = idx / (RB / 16), ch = idx % (RB / 16), tg = c * L + t;
            const bool ok = tg < p.T;
            const uint8_t* src = kbytes + (ok ? ((((size_t)b * p.T + tg) * p.H + h) * RB + 16 * ch) : 0);
            cp_async16_zf(buf + t * RS + 16 * ch, src, ok ? 16u : 0u);
        }
        const uint8_t* wsrc = ws + ((size_t)bh * NB + c) * ws_block_bytes(DK);
        for (int idx = tid; idx < (int)((WS_T + 4 * L * 4) / 16); idx += OC_THREADS)
            cp_async16_zf(buf + (size_t)L * RS + 16 * idx, wsrc + 16 * idx, 16u);
        cp_async_commit();
    };
    for (int dd = tid; dd < DK; dd += OC_THREADS) sd[dd] = p.d0 ? p.d0[(size_t)bh * DK + dd] : 1.f;
    if (NB > 0) stage(0);
#pragma unroll 1
    for (int c = 0; c < NB; ++c) {
        if (c + 1 < NB) {
            stage(c + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();   // block c's keys, T, vectors, and d
        const uint8_t* kb = smb + (c & 1) * BUF;
        const float* Tb = reinterpret_cast<const float*>(kb + (size_t)L * RS);
        const float* va = Tb + L * L;                 // a
        const float* vcR = va + L;                    // c R
        const float* vrho = va + 2 * L;               // R_{j->L}
        const float RL = va[3 * L];                   // R_L
        auto u = [&](int t, int dd) {
            const float x = to_f32(*reinterpret_cast<const Tin*>(kb + t * RS + dd * (int)sizeof(Tin)));
            return x * x;
        };
        BlockWs w = block_ws(ws, (long long)bh * NB + c, DK);
        for (int dd = tid; dd < DK; dd += OC_THREADS) w.d0[dd] = sd[dd];
        // p_t = <d, u_t>: four lanes a token; w_t = a_t - cR_t p_t
        {
            const int t = tid >> 2, part = tid & 3;
            float s = 0.f;
            for (int dd = part; dd < DK; dd += 4) s = fmaf(sd[dd], u(t, dd), s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (part == 0) sw[t] = va[t] - vcR[t] * s;
        }
        __syncthreads();
        // e = T w: four lanes a row
        {
            const int t = tid >> 2, part = tid & 3;
            float s = 0.f;
            for (int j = part; j <= t; j += 4) s = fmaf(Tb[t * L + j], sw[j], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (part == 0) {
                se[t] = s;
                w.e[t] = s;
            }
        }
        __syncthreads();
        // d <- R_L d + sum_j rho_j e_j u_j: two lanes a component
        for (int dd = tid >> 1; dd < DK; dd += OC_THREADS / 2) {
            float s = 0.f;
            for (int j = tid & 1; j < L; j += 2) s = fmaf(vrho[j] * se[j], u(j, dd), s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            if ((tid & 1) == 0) sd[dd] = fmaf(RL, sd[dd], s);
        }
        __syncthreads();   // d is final; this block's buffer may be refilled
    }
    if (p.d_out)
        for (int dd = tid; dd < DK; dd += OC_THREADS) p.d_out[(size_t)bh * DK + dd] = sd[dd];
}

// Every block at once: kw_t = (R_t d_0 + sum_{j<t} R_{j->t} e_j u_j) (.) k_t,
// the sum as a tiled product M U with M_tj = R_{j->t} e_j (j < t): thread
// (tr, tc) holds rows t = 16 a + tr and components 16 c + tc.
constexpr int OW_THREADS = 256;
template <typename Tin, int DK>
__global__ void __launch_bounds__(OW_THREADS)
osdn_write_kernel(const OsdnParams p, uint8_t* ws) {
    constexpr int NCOL = DK / 16;             // component groups a thread
    extern __shared__ float smf[];
    float* us = smf;                          // u [L][DK + 1]
    float* Ms = us + L * (DK + 1);            // M [L][LDL]
    float* sr = Ms + L * LDL;                 // r [L]
    float* se = sr + L;                       // e [L]
    float* sR = se + L;                       // R_t [L]
    float* sd = sR + L;                       // d_0 [DK]
    const int NB = (p.T + L - 1) / L;
    const long long q = blockIdx.x;
    const int bh = (int)(q / NB), c = (int)(q % NB), b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x;
    const BlockWs w = block_ws(ws, q, DK);
    load_u<Tin, DK, OW_THREADS>(p, b, h, c, us, tid);
    if (tid < L) {
        const int tg = c * L + tid;
        float rt = 1.f;
        if (tg < p.T && p.r)
            rt = to_f32(static_cast<const Tin*>(p.r)[((size_t)b * p.T + tg) * p.H + h]);
        sr[tid] = rt;
        se[tid] = __ldcg(w.e + tid);
    }
    for (int dd = tid; dd < DK; dd += OW_THREADS) sd[dd] = __ldcg(w.d0 + dd);
    __syncthreads();
    if (tid < L) {   // row t of M, and R_t
        const int t = tid;
        float rp = 1.f;
        for (int j = t - 1; j >= 0; --j) {
            Ms[t * LDL + j] = rp * se[j];
            rp *= sr[j];
        }
        for (int j = t; j < L; ++j) Ms[t * LDL + j] = 0.f;
        sR[t] = rp;
    }
    __syncthreads();
    const int tr = tid >> 4, tc = tid & 15;
    float acc[4][NCOL];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int cc = 0; cc < NCOL; ++cc) acc[a][cc] = sR[16 * a + tr] * sd[16 * cc + tc];
    // M is strictly lower triangular: the 16 columns j of segment js reach
    // only the row tiles a >= js
#pragma unroll
    for (int js = 0; js < 4; ++js) {
#pragma unroll 4
        for (int jj = 0; jj < 16; ++jj) {
            const int j = 16 * js + jj;
            float m[4], uj[NCOL];
#pragma unroll
            for (int a = js; a < 4; ++a) m[a] = Ms[(16 * a + tr) * LDL + j];
#pragma unroll
            for (int cc = 0; cc < NCOL; ++cc) uj[cc] = us[j * (DK + 1) + 16 * cc + tc];
#pragma unroll
            for (int a = js; a < 4; ++a)
#pragma unroll
                for (int cc = 0; cc < NCOL; ++cc) acc[a][cc] = fmaf(m[a], uj[cc], acc[a][cc]);
        }
    }
    const Tin* kp = static_cast<const Tin*>(p.k);
    Tin* kwp = static_cast<Tin*>(p.kw);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int t = 16 * a + tr, tg = c * L + t;
        if (tg >= p.T) continue;
        const size_t row = (((size_t)b * p.T + tg) * p.H + h) * DK;
#pragma unroll
        for (int cc = 0; cc < NCOL; ++cc)
            kwp[row + 16 * cc + tc] = from_f32<Tin>(acc[a][cc] * to_f32(kp[row + 16 * cc + tc]));
    }
}

template <typename Tin, int DK>
cudaError_t launch_dk(const OsdnParams& p, uint8_t* ws, cudaStream_t s) {
    const long long nbh = (long long)p.B * p.H;
    const int NB = (p.T + L - 1) / L;
    const size_t sm_block = ((size_t)L * (DK + 1) + 2 * (size_t)L * LDL + 3 * L + 32 * 33) * 4;
    const size_t sm_chain = chain_smem<Tin, DK>();
    const size_t sm_write = ((size_t)L * (DK + 1) + (size_t)L * LDL + 3 * L + DK) * 4;
    cudaError_t e;
    if (NB > 0) {
        auto k1 = osdn_block_kernel<Tin, DK>;
        e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_block);
        if (e != cudaSuccess) return e;
        e = launch_on(k1, dim3((unsigned)(nbh * NB)), dim3(OB_THREADS), sm_block, s, p, ws);
        if (e != cudaSuccess) return e;
    }
    auto k2 = osdn_chain_kernel<Tin, DK>;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_chain);
    if (e != cudaSuccess) return e;
    e = launch_on(k2, dim3((unsigned)nbh), dim3(OC_THREADS), sm_chain, s, p, ws);
    if (e != cudaSuccess) return e;
    if (NB > 0) {
        auto k3 = osdn_write_kernel<Tin, DK>;
        e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_write);
        if (e != cudaSuccess) return e;
        e = launch_on(k3, dim3((unsigned)(nbh * NB)), dim3(OW_THREADS), sm_write, s, p, ws);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t osdn_precondition_workspace_bytes(int B, int T, int H, int Dk) {
    const int NB = (T + L - 1) / L;
    return (size_t)B * H * NB * ws_block_bytes(Dk);
}

cudaError_t launch_osdn_precondition(const OsdnParams& p, int Dk, bool bf16, uint8_t* ws,
                                     cudaStream_t s, int* launches) {
    *launches = p.T > 0 ? 3 : 1;
    if (bf16) return Dk == 64 ? launch_dk<__nv_bfloat16, 64>(p, ws, s) : launch_dk<__nv_bfloat16, 128>(p, ws, s);
    return Dk == 64 ? launch_dk<float, 64>(p, ws, s) : launch_dk<float, 128>(p, ws, s);
}

}  // namespace gdn
