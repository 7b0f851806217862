// chunk_bwd.cu -- the backward of the chunkwise gated delta rule (scalar gate or
// none; bf16 inputs, d_k = d_v = 128; fp32 gradients).
//
// The pages print no backward formula: the gradient is the derivative of the
// chunkwise forward ("Moonshot AI's New Attention Architecture: Key
// Innovations Explained", sec. 3; the WY factors of "OSDN: Improving Delta
// Rule ...", sec. 2.1), taken by hand.  Per chunk, with h the entering state,
//   A = StrictTril(diag(beta) Kbar Kbrev^T), T = (I + A)^-1,
//   W = T diag(beta) Kbar, U = T diag(beta) V, D = U - W h,
//   O = Qbar h + P D, P = Tril(Qbar Kbrev^T), h' = gamma h + Ktil^T D,
// (Kbar = Gamma K, Kbrev = K / Gamma, Qbar = Gamma Q, Ktil = (gamma / Gamma) K)
// and upstream dO, dh':
//   dD = P^T dO + Ktil dh'
//   dh = Qbar^T dO - W^T dD + gamma dh' = (gamma I + Phi^T) dh' + Qp^T dO,
// Phi = -Ktil^T W and Qp = Qbar - P W being the forward's own step-image
// operands: the adjoint state runs the transpose of the forward's affine chunk
// map from the last chunk back.  Then, inside the chunk, dU = dD, dW = -dD h^T,
// dT = dU (beta V)^T + dW (beta Kbar)^T, dA = StrictTril(-T^T dT T^T), and the
// products through P, A, Kbar, Kbrev, Qbar, Ktil give dq, dk, dv, dbeta and
// the log-decays' dG, whose reverse cumulative sum in the chunk is dg.
//
// Two launches after the forward (run in one wave, keeping every step image
// and every chunk's entering state):
//   adjoint_chain_kernel  one CTA per (batch, head), chunks from the last back:
//                         stores the adjoint of each chunk's leaving state,
//                         then dS0; the products on the tensor cores, straight
//                         from the forward's step images, the adjoint in fp32
//   chunk_bwd_kernel      one CTA per (batch, head, chunk): recomputes the
//                         chunk's A, T, W, U, D and forms every gradient of the
//                         chunk; every product as tf32 warp MMAs (m16n8k8, fp32
//                         accumulation), tiles staged by cp.async, dq and dk
//                         accumulated in registers across the products that
//                         feed them
#include <string.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace gdn {
namespace {

using sm100::sw128_offset;

constexpr int D = 128;
constexpr int C = 64;


// Warp MMAs on tf32 operands with fp32 accumulation (m16n8k8).  A 64 x N
// output is split over the 8 warps: row strip 16 (w % 4), column half
// (N / 2) (w / 4); lane (g = lane / 4, t = lane % 4) holds, for n-tile j,
// rows r0 + g and r0 + g + 8 and columns c0 + 8 j + 2 t and + 1 (element e of
// acc[j]: row r0 + g + 8 (e / 2), column c0 + 8 j + 2 t + e % 2).  Operands
// are read through accessors a(row, k), b(k, col) from shared memory.
__device__ __forceinline__ uint32_t tf32_of(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
struct Frag {
    int r0, c0, g, t;
    __device__ int row(int e) const { return r0 + g + 8 * (e >> 1); }
    __device__ int col(int j, int e) const { return c0 + 8 * j + 2 * t + (e & 1); }
};
__device__ __forceinline__ Frag frag_of(int warp, int lane, int N) {
    return Frag{16 * (warp & 3), (N / 2) * (warp >> 2), lane >> 2, lane & 3};
}
// acc (+)= A B over K (a multiple of 8)
template <int NT, typename FA, typename FB>
__device__ __forceinline__ void mma_acc(float (&acc)[NT][4], int K, const Frag& f, FA a, FB b) {
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a0 = tf32_of(a(f.r0 + f.g, k0 + f.t));
        const uint32_t a1 = tf32_of(a(f.r0 + f.g + 8, k0 + f.t));
        const uint32_t a2 = tf32_of(a(f.r0 + f.g, k0 + f.t + 4));
        const uint32_t a3 = tf32_of(a(f.r0 + f.g + 8, k0 + f.t + 4));
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int col = f.c0 + 8 * j + f.g;
            mma_16x8x8(acc[j], a0, a1, a2, a3, tf32_of(b(k0 + f.t, col)), tf32_of(b(k0 + f.t + 4, col)));
        }
    }
}
template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}
// Sums before a shared-memory atomic: over the four lanes (t) that share a
// row of the fragment (s_lo for row r0 + g, s_hi for row r0 + g + 8), and over
// the eight lanes (g) that share a column.
__device__ __forceinline__ void frag_row_add(float* dst, const Frag& f, float s_lo, float s_hi) {
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
    s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
    s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
    if (f.t == 0) {
        atomicAdd(dst + f.r0 + f.g, s_lo);
        atomicAdd(dst + f.r0 + f.g + 8, s_hi);
    }
}
__device__ __forceinline__ void frag_col_add(float* dst, const Frag& f, int col, float s) {
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    if (f.g == 0) atomicAdd(dst + col, s);
}

// ------------------------------------------------------------ adjoint chain
// The transpose of the forward's chain, on the tensor cores.  The adjoint dh
// of a chunk's leaving state maps to the adjoint of its entering state by
//     dh <- gamma (.) dh + Phi^T dh + Qp^T dO_c,
// which, on the transposed adjoint dh^T [v][d] (as the forward chain carries
// h^T), is one accumulator per chunk:
//     D = dh^T Phi   (M = 128 v, N = 128 d', K = 128 d; A = bf16 dh^T in TMEM,
//                     B = Phi straight from the forward's step image: its rows d,
//                     columns d' contiguous, are the MN-major form of B)
//       + dO^T Qp    (K = 64 r; A = the dO tile [r][v] loaded by TMA, MN-major;
//                     B = rows 128.. of the same image tile, MN-major)
//     dh^T <- gamma (.) dh^T + D          (fp32, in the state-pass registers).
// One CTA per (batch, head), chunks from the last back.  Roles:
//   warp 0      loader: [Phi ; Qp] and dO of the next two chunks (two slots),
//               gamma (a ring of four)
//   warp 1      MMA issuer: the 12 instructions of a chunk once the state pass
//               has written dh^T (named barrier AJ_BAR_H)
//   warps 2-17  state pass (lane quarter v x column quarter d): stores each
//               chunk's leaving-state adjoint, then folds in the product
// Every mbarrier wait is bounded; named barriers join warps that run the same
// number of iterations whatever happens.
struct AdjMaps {
    CUtensorMap dO;   // dO [B][T][H*D] bf16, 64 x 64 boxes, 128-byte swizzle
};
constexpr int AJ_THREADS = 32 * 18;
constexpr int AJ_ST = 2;                       // first state-pass warp
constexpr int AJ_NST = 16;
constexpr int AJ_BAR_H = 1;
constexpr uint32_t AJ_PQ = 0;                  // 2 slots of [Phi ; Qp] (2 K-blocks each)
constexpr uint32_t AJ_DO = 2 * 2 * kImgPQBlock;   // 2 slots of dO [64 r][128 v] (two blocks)
constexpr uint32_t AJ_GAM = AJ_DO + 2 * 16384;    // 4 slots of gamma [128]
constexpr uint32_t AJ_BAR = AJ_GAM + 4 * 512;
constexpr uint32_t AJ_SMEM = AJ_BAR + 256 + 1024;
enum AjBar { AJ_FULL0, AJ_FULL1, AJ_GAM0, AJ_GAM1, AJ_GAM2, AJ_GAM3, AJ_DONE0, AJ_DONE1,
             AJ_FREE0, AJ_FREE1, AJ_FINAL, AJ_NBARS };
// TMEM (512 columns): D of slot s at 128 s, bf16 dh^T of slot s at 256 + 64 s
constexpr uint32_t AJ_TM_D = 0;
constexpr uint32_t AJ_TM_H = 256;

__global__ void __launch_bounds__(AJ_THREADS, 1)
adjoint_chain_kernel(const __grid_constant__ AdjMaps maps, const BwdParams p) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + AJ_BAR);
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    const int NC = (p.T + C - 1) / C;
    int failed = 0;
    if (tid == 0) {
        for (int i = 0; i < AJ_NBARS; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        prefetch_tmap(&maps.dO);
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    auto wait = [&](int bar, uint32_t parity) {
        if (!mbar_wait(&bars[bar], parity, &failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    };
    auto img = [&](int c) { return p.images + ((size_t)bh * NC + c) * kImgBytes; };

    if (warp == 0) {
        // =========================== loader (step j = chunk NC - 1 - j)
#pragma unroll 1
        for (int j = 0; j < NC; ++j) {
            const int c = NC - 1 - j, s = j & 1;
            if (j >= 2) wait(AJ_FREE0 + s, ((j - 2) >> 1) & 1);   // the MMA of step j - 2 is done
            if (failed) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[AJ_FULL0 + s], 2 * kImgPQBlock + 16384);
                bulk_load(sm + AJ_PQ + s * 2 * kImgPQBlock, img(c) + kImgPQ, 2 * kImgPQBlock,
                          &bars[AJ_FULL0 + s]);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_3d(sm + AJ_DO + s * 16384 + blk * 8192, &maps.dO, &bars[AJ_FULL0 + s],
                                h * D + 64 * blk, c * C, b);
                mbar_arrive_expect_tx(&bars[AJ_GAM0 + (j & 3)], 512);
                bulk_load(sm + AJ_GAM + (j & 3) * 512, img(c) + kImgGam, 512, &bars[AJ_GAM0 + (j & 3)]);
            }
        }
    } else if (warp == 1) {
        // =========================== MMA issuer
        const bool leader = lane == 0;
        const uint32_t id_h = idesc_bf16_f32(128, 128, false, true);   // A in TMEM, B MN-major
        const uint32_t id_o = idesc_bf16_f32(128, 128, true, true);    // A, B MN-major
#pragma unroll 1
        for (int j = 0; j < NC; ++j) {
            const int s = j & 1;
            wait(AJ_FULL0 + s, (j >> 1) & 1);
            named_bar(AJ_BAR_H, 32 + 32 * AJ_NST);   // dh^T of step j is in TMEM
            tc_fence_after();
            if (leader && !failed) {
                const uint32_t pq = sb + AJ_PQ + s * 2 * kImgPQBlock;
                const uint32_t dO = sb + AJ_DO + s * 16384;
#pragma unroll
                for (int k = 0; k < 8; ++k)   // dh^T Phi: K = d, rows d of Phi at 128 B
                    mma_bf16_ta(tmem + AJ_TM_D + 128 * s, tmem + AJ_TM_H + 64 * s + 8 * k,
                                sdesc_sw128(pq + k * 2048, kImgPQBlock, 1024), id_h, k > 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // dO^T Qp: K = r, Qp rows 128 + r
                    mma_bf16(tmem + AJ_TM_D + 128 * s, sdesc_sw128(dO + k * 2048, 8192, 1024),
                             sdesc_sw128(pq + 16384 + k * 2048, kImgPQBlock, 1024), id_o, true);
                mma_commit(&bars[AJ_DONE0 + s]);
                mma_commit(&bars[AJ_FREE0 + s]);
            }
            __syncwarp();
        }
        if (leader) mma_commit(&bars[AJ_FINAL]);
        int f2 = 0;
        if (!mbar_wait(&bars[AJ_FINAL], 0, &f2)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    } else {
        // =========================== state pass: dh^T row v, columns d = 32 cq ..
        const int v = (warp & 3) * 32 + lane;
        const int cq = (warp - AJ_ST) >> 2;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        float dh[32];
        {
            const float* src = p.dS ? p.dS + (size_t)bh * D * D + (size_t)(32 * cq) * D + v : nullptr;
#pragma unroll
            for (int e = 0; e < 32; ++e) dh[e] = src ? __ldcg(src + (size_t)e * D) : 0.f;
        }
        // dh <- gamma_j (.) dh + D_j, once the product of step j is done
        auto fold = [&](int j) {
            wait(AJ_GAM0 + (j & 3), (j >> 2) & 1);
            const float* gp = reinterpret_cast<const float*>(sm + AJ_GAM + (j & 3) * 512) + 32 * cq;
            wait(AJ_DONE0 + (j & 1), (j >> 1) & 1);
            tc_fence_after();
            float x[32];
            tmem_ld32(tmem + AJ_TM_D + 128 * (j & 1) + lane_off + 32 * cq, x);
            tmem_wait_ld();
            reg_fence(x);
#pragma unroll
            for (int e = 0; e < 32; ++e) dh[e] = fmaf(gp[e], dh[e], x[e]);
        };
#pragma unroll 1
        for (int j = 0; j < NC; ++j) {
            const int c = NC - 1 - j;
            if (j > 0) fold(j - 1);
            // the adjoint of chunk c's leaving state
            float* dst = p.dh_all + ((size_t)bh * NC + c) * D * D + (size_t)(32 * cq) * D + v;
#pragma unroll
            for (int e = 0; e < 32; ++e) dst[(size_t)e * D] = dh[e];
            float pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                __nv_bfloat162 t2 = __floats2bfloat162_rn(dh[2 * e], dh[2 * e + 1]);
                pk[e] = __uint_as_float(*reinterpret_cast<uint32_t*>(&t2));
            }
            tmem_st16(tmem + AJ_TM_H + 64 * (j & 1) + 16 * cq + lane_off, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            named_bar_arrive(AJ_BAR_H, 32 + 32 * AJ_NST);
        }
        if (NC > 0) fold(NC - 1);
        if (p.dS0) {
            float* dst = p.dS0 + (size_t)bh * D * D + (size_t)(32 * cq) * D + v;
#pragma unroll
            for (int e = 0; e < 32; ++e) dst[(size_t)e * D] = dh[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------- chunk backward
// 16-byte copies global -> shared that bypass the registers (L2 only), so a
// thread issues all of its copies of a tile before waiting once; a source size
// of 0 fills the 16 bytes with zeros (rows past the end of the sequence).
__device__ __forceinline__ void cpa16(void* dst, const void* src, uint32_t src_bytes = 16u) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sm100::smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cpa_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

constexpr int CB_THREADS = 256;
constexpr int LDM = D + 4;   // fp32 row stride of [64][128] matrices
constexpr int LDS = C + 1;   // fp32 row stride of [64][64] matrices
// bf16 [64][LDB] tiles: rows padded to 136 elements (272 B), so that reading a
// column (16 rows, one element each) touches 8 banks instead of one
constexpr int LDB = D + 8;
constexpr uint32_t BW_TILE = C * LDB * 2;
constexpr uint32_t BW_Q = 0, BW_K = BW_TILE, BW_V = 2 * BW_TILE, BW_DO = 3 * BW_TILE;
constexpr uint32_t BW_STAGE = 4 * BW_TILE;                                // [64][LDM] fp32
constexpr uint32_t BW_P = BW_STAGE + C * LDM * 4;                         // [64][LDS]
constexpr uint32_t BW_T = BW_P + C * LDS * 4;
constexpr uint32_t BW_A = BW_T + C * LDS * 4;
constexpr uint32_t BW_MD = BW_A + C * LDS * 4;                            // [64][LDM]
constexpr uint32_t BW_MW = BW_MD + C * LDM * 4;
constexpr uint32_t BW_VEC = BW_MW + C * LDM * 4;                          // vectors
constexpr uint32_t BW_SMEM = BW_VEC + 8 * C * 4 + 1024;
static_assert(BW_SMEM <= 232448, "chunk backward shared memory");

template <bool GATED>
__global__ void __launch_bounds__(CB_THREADS, 1)
chunk_bwd_kernel(const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const __nv_bfloat16* sQ = reinterpret_cast<const __nv_bfloat16*>(sm + BW_Q);
    const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(sm + BW_K);
    const __nv_bfloat16* sV = reinterpret_cast<const __nv_bfloat16*>(sm + BW_V);
    const __nv_bfloat16* sdO = reinterpret_cast<const __nv_bfloat16*>(sm + BW_DO);
    float* stage = reinterpret_cast<float*>(sm + BW_STAGE);
    float* sP = reinterpret_cast<float*>(sm + BW_P);
    float* sT = reinterpret_cast<float*>(sm + BW_T);
    float* sA = reinterpret_cast<float*>(sm + BW_A);
    float* MD = reinterpret_cast<float*>(sm + BW_MD);
    float* MW = reinterpret_cast<float*>(sm + BW_MW);
    float* sG = reinterpret_cast<float*>(sm + BW_VEC);   // G (in-chunk log-decay cumsum)
    float* sGam = sG + C;                                // Gamma = e^G
    float* sBeta = sG + 2 * C;
    float* sdG = sG + 3 * C;
    float* sdB = sG + 4 * C;                             // dbeta
    float* sRed = sG + 5 * C;                            // a reduction slot

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int NC = (p.T + C - 1) / C;
    const int item = blockIdx.x, bh = item / NC, c = item % NC;
    const int b = bh / p.H, h = bh % p.H;
    auto tok = [&](int r) { return ((size_t)b * p.T + (size_t)c * C + r) * p.H + h; };
    const int n = min(C, p.T - c * C);

    // ---- inputs of the chunk (rows past the sequence end are zero-filled; their
    // copies read nothing and name row 0, which exists)
    for (int idx = tid; idx < 4 * C * D / 8; idx += CB_THREADS) {
        const int m = idx / (C * D / 8), rem = idx % (C * D / 8), r = rem >> 4, j = rem & 15;
        const __nv_bfloat16* src = m == 0 ? static_cast<const __nv_bfloat16*>(p.q)
                                   : m == 1 ? static_cast<const __nv_bfloat16*>(p.k)
                                   : m == 2 ? static_cast<const __nv_bfloat16*>(p.v)
                                            : static_cast<const __nv_bfloat16*>(p.dO);
        cpa16(sm + m * BW_TILE + r * LDB * 2 + 16 * j, src + tok(r < n ? r : 0) * D + 8 * j,
              r < n ? 16u : 0u);
    }
    cpa_wait_all();
    if (tid < C) {
        float bt = 0.f, gv = 0.f;
        if (tid < n) {
            bt = __bfloat162float(static_cast<const __nv_bfloat16*>(p.beta)[tok(tid)]);
            if (GATED) gv = __bfloat162float(static_cast<const __nv_bfloat16*>(p.g)[tok(tid)]);
        }
        sBeta[tid] = bt;
        sG[tid] = gv;
        sdG[tid] = 0.f;
        sdB[tid] = 0.f;
    }
    __syncthreads();
    if (warp == 0) {   // in-chunk cumulative sum of g (two tokens a lane)
        const float a0 = sG[2 * lane], a1 = sG[2 * lane + 1];
        float incl = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        float excl = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) excl = 0.f;
        sG[2 * lane] = excl + a0;
        sG[2 * lane + 1] = incl;
        sGam[2 * lane] = __expf(excl + a0);
        sGam[2 * lane + 1] = __expf(incl);
    }
    __syncthreads();
    const float Glast = sG[C - 1], gamma = sGam[C - 1];
    auto E = [&](int r, int i) { return i <= r ? __expf(sG[r] - sG[i]) : 0.f; };
    auto kf = [&](int r, int d) { return __bfloat162float(sK[r * LDB + d]); };
    auto qf = [&](int r, int d) { return __bfloat162float(sQ[r * LDB + d]); };
    auto vf = [&](int r, int d) { return __bfloat162float(sV[r * LDB + d]); };
    auto of = [&](int r, int d) { return __bfloat162float(sdO[r * LDB + d]); };
    const Frag F64 = frag_of(warp, lane, C), F128 = frag_of(warp, lane, D);

    // ---- P = Tril(E (.) Q K^T), A = StrictTril(beta_r E (.) K K^T)
    {
        float aq[4][4], ak[4][4];
        zero(aq);
        zero(ak);
        mma_acc<4>(aq, D, F64, qf, [&](int d, int i) { return kf(i, d); });
        mma_acc<4>(ak, D, F64, kf, [&](int d, int i) { return kf(i, d); });
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F64.row(e), i = F64.col(j, e);
                const float ev = E(r, i);
                sP[r * LDS + i] = ev * aq[j][e];
                sA[r * LDS + i] = i < r ? sBeta[r] * ev * ak[j][e] : 0.f;
            }
    }
    __syncthreads();
    // ---- T = (I + A)^-1 by forward substitution, one column a thread
    if (tid < C) {
        const int col = tid;
        for (int r = 0; r < C; ++r) {
            float x = (r == col) ? 1.f : 0.f;
            if (r > col) {
                for (int i = col; i < r; ++i) x = fmaf(-sA[r * LDS + i], sT[i * LDS + col], x);
            }
            sT[r * LDS + col] = r >= col ? x : 0.f;
        }
    }
    __syncthreads();
    // ---- W = T diag(beta Gamma) K, U = T diag(beta) V
    {
        float aw[8][4], au[8][4];
        zero(aw);
        zero(au);
        mma_acc<8>(aw, C, F128, [&](int r, int i) { return sT[r * LDS + i] * sBeta[i] * sGam[i]; }, kf);
        mma_acc<8>(au, C, F128, [&](int r, int i) { return sT[r * LDS + i] * sBeta[i]; }, vf);
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F128.row(e), v = F128.col(j, e);
                MW[r * LDM + v] = aw[j][e];
                MD[r * LDM + v] = au[j][e];
            }
    }
    // ---- D = U - W h (h staged by halves of 64 rows)
    const float* hsrc = p.h_all + ((size_t)bh * NC + c) * D * D;
    const float* dhsrc = p.dh_all + ((size_t)bh * NC + c) * D * D;
    auto stage_half = [&](const float* src, int half) {
        __syncthreads();
#pragma unroll
        for (int idx = 4 * tid; idx < C * D; idx += 4 * CB_THREADS)
            cpa16(stage + (idx >> 7) * LDM + (idx & 127), src + (size_t)half * C * D + idx);
        cpa_wait_all();
        __syncthreads();
    };
    {
        float ad[8][4];
        zero(ad);
        for (int half = 0; half < 2; ++half) {
            stage_half(hsrc, half);
            mma_acc<8>(ad, C, F128, [&](int r, int d) { return MW[r * LDM + 64 * half + d]; },
                       [&](int d, int v) { return stage[d * LDM + v]; });
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F128.row(e), v = F128.col(j, e);
                MD[r * LDM + v] -= ad[j][e];
            }
    }
    __syncthreads();
    // dq and dk of this thread's fragment elements (rows r, columns d of the
    // 64 x 128 layout), summed over every product below
    float dq[8][4], dk[8][4];
    zero(dq);
    zero(dk);
    // ---- dD = P^T dO + Ktil dh' (into MW, W being dead), dKtil = D dh'^T,
    //      <h, dh'>; dh' staged by halves of 64 rows (d)
    {
        float add[8][4];
        zero(add);
        mma_acc<8>(add, C, F128, [&](int i, int r) { return sP[r * LDS + i]; }, of);
        float hdh = 0.f, lastsum = 0.f;   // <h, dh'>; the K~ terms of dG_last
        for (int half = 0; half < 2; ++half) {
            stage_half(dhsrc, half);
            // Ktil[i][d] = k_id e^(Glast - G_i), d in this half
            mma_acc<8>(add, C, F128,
                       [&](int i, int d) { return kf(i, 64 * half + d) * __expf(Glast - sG[i]); },
                       [&](int d, int v) { return stage[d * LDM + v]; });
            // dKtil[i][d] = sum_v D[i][v] dh'[d][v] for the columns d of this
            // half: the warps that own them in the 64 x 128 layout
            if ((warp >> 2) == half) {
                float akt[8][4];
                zero(akt);
                mma_acc<8>(akt, D, F128, [&](int i, int v) { return MD[i * LDM + v]; },
                           [&](int v, int d) { return stage[(d - 64 * half) * LDM + v]; });
                float lo = 0.f, hi = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = F128.row(e), d = F128.col(j, e);
                        const float f = __expf(Glast - sG[i]);
                        dk[j][e] = fmaf(akt[j][e], f, dk[j][e]);
                        const float part = akt[j][e] * kf(i, d) * f;
                        if (e < 2) lo += part;
                        else hi += part;
                    }
                frag_row_add(sdG, F128, -lo, -hi);
                lastsum += lo + hi;
            }
#pragma unroll 4
            for (int idx = 4 * tid; idx < C * D; idx += 4 * CB_THREADS) {
                const float4 hv = __ldcg(reinterpret_cast<const float4*>(hsrc + (size_t)half * C * D + idx));
                const float* sp = stage + (idx >> 7) * LDM + (idx & 127);
                hdh = fmaf(hv.x, sp[0], hdh);
                hdh = fmaf(hv.y, sp[1], hdh);
                hdh = fmaf(hv.z, sp[2], hdh);
                hdh = fmaf(hv.w, sp[3], hdh);
            }
        }
        // <h, dh'> over the block, into dG_last (gamma <h, dh'>)
        float last = gamma * hdh + lastsum;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) last += __shfl_xor_sync(0xffffffffu, last, off);
        if (lane == 0) atomicAdd(&sdG[C - 1], last);
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) MW[F128.row(e) * LDM + F128.col(j, e)] = add[j][e];   // dD
    }
    __syncthreads();
    // ---- dP = Tril(dO D^T); tP = dP (.) P -> dG; dPE = dP (.) E into sP
    {
        float adp[4][4];
        zero(adp);
        mma_acc<4>(adp, D, F64, of, [&](int v, int i) { return MD[i * LDM + v]; });
        float lo = 0.f, hi = 0.f, colp[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) colp[j][0] = colp[j][1] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F64.row(e), i = F64.col(j, e);
                const float t = i <= r ? adp[j][e] * sP[r * LDS + i] : 0.f;
                if (e < 2) lo += t;
                else hi += t;
                colp[j][e & 1] += t;
            }
        frag_row_add(sdG, F64, lo, hi);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < 2; ++q) frag_col_add(sdG, F64, F64.c0 + 8 * j + 2 * F64.t + q, -colp[j][q]);
        __syncthreads();   // every thread has read P
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F64.row(e), i = F64.col(j, e);
                sP[r * LDS + i] = i <= r ? adp[j][e] * E(r, i) : 0.f;
            }
    }
    __syncthreads();
    // dq_r += sum_i dPE_ri k_i;  dk_i += sum_r dPE_ri q_r
    mma_acc<8>(dq, C, F128, [&](int r, int i) { return sP[r * LDS + i]; }, kf);
    mma_acc<8>(dk, C, F128, [&](int i, int r) { return sP[r * LDS + i]; }, qf);
    // ---- dQbar = dO h^T -> dq += Gamma dQbar, dG_r += Gamma_r <dQbar_r, q_r>;
    //      dW = -dD h^T (into MD, D being dead from here); h by halves of 64
    //      rows d, each half's columns by the warps that own them
    for (int half = 0; half < 2; ++half) {
        stage_half(hsrc, half);
        if ((warp >> 2) == half) {
            float t1[8][4], t2[8][4];
            zero(t1);
            zero(t2);
            mma_acc<8>(t1, D, F128, of, [&](int v, int d) { return stage[(d - 64 * half) * LDM + v]; });
            mma_acc<8>(t2, D, F128, [&](int r, int v) { return MW[r * LDM + v]; },
                       [&](int v, int d) { return stage[(d - 64 * half) * LDM + v]; });
            float lo = 0.f, hi = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = F128.row(e), d = F128.col(j, e);
                    dq[j][e] = fmaf(sGam[r], t1[j][e], dq[j][e]);
                    const float part = sGam[r] * t1[j][e] * qf(r, d);
                    if (e < 2) lo += part;
                    else hi += part;
                    t2[j][e] = -t2[j][e];
                }
            frag_row_add(sdG, F128, lo, hi);
            // every warp of this half has read MD's D values (the dP product
            // above, behind a barrier): dW may overwrite them
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) MD[F128.row(e) * LDM + F128.col(j, e)] = t2[j][e];
        }
    }
    __syncthreads();
    // ---- dv = beta T^T dU (dU = dD);  dbeta += <T^T dU, V> + <T^T dW, Kbar>;
    //      dKbar = beta T^T dW -> dk += Gamma dKbar, dG += <dKbar, Kbar>
    {
        float tu[8][4], tw[8][4];
        zero(tu);
        zero(tw);
        mma_acc<8>(tu, C, F128, [&](int r, int i) { return sT[i * LDS + r]; },
                   [&](int i, int v) { return MW[i * LDM + v]; });
        mma_acc<8>(tw, C, F128, [&](int r, int i) { return sT[i * LDS + r]; },
                   [&](int i, int v) { return MD[i * LDM + v]; });
        float db_lo = 0.f, db_hi = 0.f, dg_lo = 0.f, dg_hi = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F128.row(e), v = F128.col(j, e);
                if (r < n) p.dv[tok(r) * D + v] = sBeta[r] * tu[j][e];
                const float kbar = sGam[r] * kf(r, v);
                const float db = fmaf(tu[j][e], vf(r, v), tw[j][e] * kbar);
                const float dkb = sBeta[r] * tw[j][e];
                dk[j][e] = fmaf(sGam[r], dkb, dk[j][e]);
                const float dg = dkb * kbar;
                if (e < 2) {
                    db_lo += db;
                    dg_lo += dg;
                } else {
                    db_hi += db;
                    dg_hi += dg;
                }
            }
        frag_row_add(sdB, F128, db_lo, db_hi);
        frag_row_add(sdG, F128, dg_lo, dg_hi);
    }
    // ---- dT = dD (beta V)^T + dW (beta Kbar)^T  (into sA);  tmp = T^T dT  (into stage)
    {
        float adt[4][4];
        zero(adt);
        mma_acc<4>(adt, D, F64, [&](int r, int v) { return MW[r * LDM + v]; },
                   [&](int v, int i) { return sBeta[i] * vf(i, v); });
        mma_acc<4>(adt, D, F64, [&](int r, int d) { return MD[r * LDM + d]; },
                   [&](int d, int i) { return sBeta[i] * sGam[i] * kf(i, d); });
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sA[F64.row(e) * LDS + F64.col(j, e)] = adt[j][e];
    }
    __syncthreads();
    {
        float at[4][4];
        zero(at);
        mma_acc<4>(at, C, F64, [&](int r, int i) { return sT[i * LDS + r]; },
                   [&](int i, int j) { return sA[i * LDS + j]; });
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) stage[F64.row(e) * LDS + F64.col(j, e)] = at[j][e];
    }
    __syncthreads();
    // ---- dA = StrictTril(-tmp T^T); dKK = beta_r dA; dbeta += sum_i dA KKE;
    //      dKKE = dKK (.) E into sA; KKE recomputed (E (.) K K^T)
    {
        float ada[4][4], akk[4][4];
        zero(ada);
        zero(akk);
        mma_acc<4>(ada, C, F64, [&](int r, int i) { return stage[r * LDS + i]; },
                   [&](int i, int j) { return sT[j * LDS + i]; });
        mma_acc<4>(akk, D, F64, kf, [&](int d, int i) { return kf(i, d); });
        __syncthreads();
        float db_lo = 0.f, db_hi = 0.f, ra_lo = 0.f, ra_hi = 0.f, cola[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) cola[j][0] = cola[j][1] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = F64.row(e), i = F64.col(j, e);
                float val = 0.f;
                if (i < r) {
                    const float dA = -ada[j][e];
                    const float ev = E(r, i);
                    const float db = dA * ev * akk[j][e];
                    const float dkke = sBeta[r] * dA * ev;
                    const float t = dkke * akk[j][e];
                    if (e < 2) {
                        db_lo += db;
                        ra_lo += t;
                    } else {
                        db_hi += db;
                        ra_hi += t;
                    }
                    cola[j][e & 1] += t;
                    val = dkke;
                }
                sA[r * LDS + i] = val;
            }
        frag_row_add(sdB, F64, db_lo, db_hi);
        frag_row_add(sdG, F64, ra_lo, ra_hi);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int q = 0; q < 2; ++q) frag_col_add(sdG, F64, F64.c0 + 8 * j + 2 * F64.t + q, -cola[j][q]);
    }
    __syncthreads();
    // dk_r += sum_i dKKE_ri k_i;  dk_i += sum_r dKKE_ri k_r
    mma_acc<8>(dk, C, F128, [&](int r, int i) { return sA[r * LDS + i]; }, kf);
    mma_acc<8>(dk, C, F128, [&](int i, int r) { return sA[r * LDS + i]; }, kf);
    __syncthreads();
    // ---- outputs: dq, dk (this thread's elements, two adjacent columns a
    // store), dbeta, dg (reverse cumsum of dG)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = F128.row(2 * h2), d = F128.col(j, 0);
            if (r < n) {
                *reinterpret_cast<float2*>(p.dq + tok(r) * D + d) = make_float2(dq[j][2 * h2], dq[j][2 * h2 + 1]);
                *reinterpret_cast<float2*>(p.dk + tok(r) * D + d) = make_float2(dk[j][2 * h2], dk[j][2 * h2 + 1]);
            }
        }
    if (warp == 0) {   // dg_t = sum_{r >= t} dG_r: a reverse scan, two tokens a lane
        const int r0 = C - 2 - 2 * lane;     // lane 0 takes the last two tokens
        const float a1 = sdG[r0 + 1], a0 = sdG[r0];
        float incl = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        float excl = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) excl = 0.f;
        const float g1 = excl + a1, g0 = incl;
        if (GATED && p.dg) {
            if (r0 + 1 < n) p.dg[tok(r0 + 1)] = g1;
            if (r0 < n) p.dg[tok(r0)] = g0;
        }
        if (r0 + 1 < n) p.dbeta[tok(r0 + 1)] = sdB[r0 + 1];
        if (r0 < n) p.dbeta[tok(r0)] = sdB[r0];
    }
    (void)sRed;
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H) {
    const int NC = (T + C - 1) / C;
    if (NC == 0 || B == 0 || H == 0) return 0;
    const size_t nbh = (size_t)B * H;
    const size_t fwd = chunk_fwd_tc_capture_bytes(B, T, H);
    const size_t o = ((size_t)B * T * H * D * 2 + 255) & ~(size_t)255;
    return fwd + o + 2 * nbh * NC * D * D * sizeof(float);
}

cudaError_t launch_chunk_bwd(const ChunkParams& pf, const BwdParams& pb0, int gate,
                             uint8_t* ws, size_t ws_bytes, cudaStream_t s, int* launches) {
    *launches = 0;
    const int NC = (pf.T + C - 1) / C;
    const size_t nbh = (size_t)pf.B * pf.H;
    const size_t fwd = chunk_fwd_tc_capture_bytes(pf.B, pf.T, pf.H);
    const size_t o_bytes = ((size_t)pf.B * pf.T * pf.H * D * 2 + 255) & ~(size_t)255;
    if (ws_bytes < chunk_bwd_workspace_bytes(pf.B, pf.T, pf.H)) return cudaErrorInvalidValue;
    BwdParams pb = pb0;
    pb.images = ws;
    pb.h_all = reinterpret_cast<float*>(ws + fwd + o_bytes);
    pb.dh_all = pb.h_all + nbh * NC * D * D;
    // 1. the forward in one wave, keeping the images and every entering state
    ChunkParams p = pf;
    p.ws = ws;
    p.o = ws + fwd;
    p.s_out = nullptr;
    int nf = 0;
    cudaError_t e = launch_chunk_fwd_tc_capture(p, gate, fwd, pb.h_all, s, &nf);
    *launches += nf;
    if (e != cudaSuccess) return e;
    // 2. the adjoint state, chunks from the last back
    AdjMaps am;
    memset(&am, 0, sizeof(am));
    {
        const uint64_t dims[3] = {(uint64_t)pf.H * D, (uint64_t)pf.T, (uint64_t)pf.B};
        const uint64_t strides[2] = {(uint64_t)pf.H * D * 2, (uint64_t)pf.T * pf.H * D * 2};
        const uint32_t box[3] = {64, 64, 1};
        if (!make_tmap_bf16(&am.dO, pb.dO, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    e = cudaFuncSetAttribute(adjoint_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)AJ_SMEM);
    if (e != cudaSuccess) return e;
    e = launch_on(adjoint_chain_kernel, dim3((unsigned)nbh), dim3(AJ_THREADS), AJ_SMEM, s, am, pb);
    if (e != cudaSuccess) return e;
    ++*launches;
    // 3. every chunk's gradients
    auto kern = gate == kGateScalar ? chunk_bwd_kernel<true> : chunk_bwd_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BW_SMEM);
    if (e != cudaSuccess) return e;
    e = launch_on(kern, dim3((unsigned)(nbh * NC)), dim3(CB_THREADS), BW_SMEM, s, pb);
    if (e != cudaSuccess) return e;
    ++*launches;
    return cudaSuccess;
}

}  // namespace gdn
