// chunk_fwd_tc.cu -- chunkwise gated delta rule on the sm_100a tensor cores
// (bf16 operands, fp32 accumulation in TMEM, fp32 state), d_k = d_v = 128.
//
// The chunkwise algorithm of "Moonshot AI's New Attention Architecture: Key
// Innovations Explained" (sec. 3, state recurrence and causal output) with the
// UT/WY transform of "OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention" (sec. 2.1, chunk Gram matrix + WY),
// for a scalar (or no) forget gate.  Per chunk of C = 64 tokens, h the
// entering state M = S^T [d_k][d_v], G the in-chunk log-decay cumsum:
//   S  = [K; Q] K^T                 (one 128-row MMA: K K^T and Q K^T)
//   A  = StrictTril(beta_r e^(G_r-G_i) (K K^T)_ri),  P = Tril(e^(G_r-G_i) (Q K^T)_ri)
//   T  = (I + A)^-1                 (blocked forward substitution)
//   [0; W] = [0; T diag(beta e^G)] K
//   X  = [T diag(beta); 0] V        = [U; 0]
//   X += [-W; Q_bar] h              -> rows 0..63: D = U - W h, rows 64..127: Q_bar h
//   X += [0; P] D                   -> rows 64..127: O = Q_bar h + P D
//   h  = e^(G_C) h + K^T (diag(e^(G_C - G_i)) D)
// Every product is a tcgen05.mma with M = 128; operands live in 128 B-swizzled
// shared memory: the K/Q/V tiles exactly as TMA loads them (K-major when the
// tokens are rows, MN-major when they are the reduction dimension), the other
// operands written in the same canonical layouts.
//
// Two kernels per wave of chunks:
//   chunk_prep_tc_kernel  one CTA per chunk, fully parallel: gates, S, A, P,
//                         T, and the bf16 operands T diag(beta),
//                         T diag(beta e^G), P plus the gate factors, written
//                         to the workspace as the exact shared-memory image
//                         the chain kernel uses (the wave is sized so the
//                         workspace stays in L2);
//   chunk_fwd_tc_kernel   one CTA per (batch, head), the serial state chain:
//                         bulk-copies the prep images, W / U products, the
//                         c- and d-products, state and output, with warp roles
//                         chain (0-3), stager (4-7) and control (8) handing
//                         over through mbarriers.
// Every mbarrier wait is bounded; a wait that gives up sets the library status
// word and the kernel winds down without further waits.
#include "common.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NPR = 256;         // prep kernel threads (8 warps)
constexpr int LDF = 72;          // fp32 row stride of the A / T scratch (conflict-free mma fragments)
constexpr int GATE_FLOATS = 7 * 64;   // G, e^G, e^(G_C-G), beta, u, w, flag

// Workspace image of one chunk (bytes).
constexpr uint32_t WS_TU = 0;          // T diag(beta), K-major [64 r][64 i], swizzled
constexpr uint32_t WS_TW = 8192;       // T diag(beta e^G)
constexpr uint32_t WS_P = 16384;       // P
constexpr uint32_t WS_FAC = 24576;     // e^G [64], e^(G_C - G) [64] (fp32)
constexpr uint32_t WS_CHUNK = WS_FAC + 2 * 64 * 4;
constexpr size_t WAVE_BYTES = size_t(32) << 20;   // workspace per wave (kept L2-resident)

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ void st_row_chunk(uint8_t* tile, int row, int j, const float* v,
                                             float scale) {
    uint4 w;
    w.x = pack_bf16(v[0] * scale, v[1] * scale);
    w.y = pack_bf16(v[2] * scale, v[3] * scale);
    w.z = pack_bf16(v[4] * scale, v[5] * scale);
    w.w = pack_bf16(v[6] * scale, v[7] * scale);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, 8 * j)) = w;
}

__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int N>
__device__ __forceinline__ void ld_cols(uint32_t addr, float (&v)[N]) {
    static_assert(N % 16 == 0, "");
#pragma unroll
    for (int j = 0; j < N / 16; ++j)
        tmem_ld16(addr + 16 * j, *reinterpret_cast<float(*)[16]>(v + 16 * j));
    tmem_wait_ld();
    reg_fence(v);
}

template <int N>
__device__ __forceinline__ void st_cols(uint32_t addr, float (&v)[N]) {
#pragma unroll
    for (int j = 0; j < N / 16; ++j)
        tmem_st16(addr + 16 * j, *reinterpret_cast<float(*)[16]>(v + 16 * j));
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// d (16 x 8, fp32) += a (16 x 8) * b (8 x 8), warp-level tensor-core MMA on tf32
// operands.  Fragments (g = lane / 4, t = lane % 4): a0 (g, t), a1 (g + 8, t),
// a2 (g, t + 4), a3 (g + 8, t + 4); b0 (k = t, n = g), b1 (k = t + 4, n = g);
// d0 (g, 2t), d1 (g, 2t + 1), d2 (g + 8, 2t), d3 (g + 8, 2t + 1).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const float* M, int r0, int k0,
                                                const float* N, int kn0, int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t a0 = to_tf32(M[(r0 + g) * LDF + k0 + t]);
    const uint32_t a1 = to_tf32(M[(r0 + g + 8) * LDF + k0 + t]);
    const uint32_t a2 = to_tf32(M[(r0 + g) * LDF + k0 + t + 4]);
    const uint32_t a3 = to_tf32(M[(r0 + g + 8) * LDF + k0 + t + 4]);
    const uint32_t b0 = to_tf32(N[(kn0 + t) * LDF + n0 + g]);
    const uint32_t b1 = to_tf32(N[(kn0 + t + 4) * LDF + n0 + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void store_16x8(float* X, int r0, int n0, const float (&d)[4], float s,
                                           int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(X + (r0 + g) * LDF + n0 + 2 * t) = make_float2(s * d[0], s * d[1]);
    *reinterpret_cast<float2*>(X + (r0 + g + 8) * LDF + n0 + 2 * t) = make_float2(s * d[2], s * d[3]);
}

// T = (I + A)^-1 for strictly lower-triangular A (64 x 64, fp32), 256 threads
// (8 warps).  (1) the four diagonal 16 x 16 inverses by right-looking
// substitution on CUDA cores, one column per thread; (2) 16 -> 32:
// T_10 = -T_11 (A_10 T_00) for the two diagonal 32 x 32 blocks; (3) 32 -> 64:
// the same with 32 x 32 blocks.  The block products run as warp MMAs on tf32
// operands with fp32 accumulation (T is rounded to bf16 right after, so the
// tf32 operand rounding stays well below that); the inner product X goes
// through the strictly upper part of Tm, which T never uses.
__device__ __forceinline__ void forward_substitution(const float* A, float* Tm, int pt) {
    const int lane = pt & 31, w = pt >> 5;
    if (pt < 64) {
        const int o = 16 * (pt >> 4), c = pt & 15;
        float p[16], x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) p[r] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            x[i] = (i == c) ? 1.f : (i < c ? 0.f : -p[i]);
#pragma unroll
            for (int r = i + 1; r < 16; ++r) p[r] = fmaf(A[(o + r) * LDF + o + i], x[i], p[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(o + r) * LDF + o + c] = x[r];
    }
    named_bar(2, NPR);
    if (w < 4) {   // 16 -> 32: pair pr, n-tile nt of the 16 x 16 block (2pr+1, 2pr)
        const int pr = w >> 1, nt = w & 1;
        const int ri = 16 * (2 * pr + 1), cj = 16 * (2 * pr);
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) mma_tf32_16x8x8(d, A, ri, cj + 8 * ks, Tm, cj + 8 * ks, cj + 8 * nt, lane);
        store_16x8(Tm, cj, ri + 8 * nt, d, 1.f, lane);       // X in the upper block (cj, ri)
        __syncwarp();
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) mma_tf32_16x8x8(e, Tm, ri, ri + 8 * ks, Tm, cj + 8 * ks, ri + 8 * nt, lane);
        store_16x8(Tm, ri, cj + 8 * nt, e, -1.f, lane);
    }
    named_bar(2, NPR);
    const int rt = w >> 2, nt = w & 3;    // 32 -> 64: row tile rt (16 rows), n-tile nt (8 cols)
    {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            if (8 * ks + 7 >= 8 * nt)      // rows of T32_00 above its diagonal are zero
                mma_tf32_16x8x8(d, A, 32 + 16 * rt, 8 * ks, Tm, 8 * ks, 8 * nt, lane);
        store_16x8(Tm, 16 * rt, 32 + 8 * nt, d, 1.f, lane);  // X in the upper-right quadrant
    }
    named_bar(2, NPR);
    {
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            if (8 * ks <= 16 * rt + 15)    // columns of T32_11 right of its diagonal are zero
                mma_tf32_16x8x8(e, Tm + 32, 32 + 16 * rt, 8 * ks, Tm + 32, 8 * ks, 8 * nt, lane);
        store_16x8(Tm, 32 + 16 * rt, 8 * nt, e, -1.f, lane);
    }
    named_bar(2, NPR);
}


// In-chunk gates for one scalar-gated chunk, by one warp: inclusive scan of g
// (two tokens per lane), e^G, e^(G_C - G), and the factors u_r = e^(G_r - G_31),
// w_i = e^(G_31 - G_i) with e^(G_r - G_i) = u_r w_i, usable while each half of
// the chunk decays by less than e^80, so that every factor and its reciprocal
// stay normal fp32 numbers (flag).  gbuf[0..63] holds g on entry.
template <int GATE>
__device__ __forceinline__ void chunk_gates(float* gbuf, int lane) {
    if constexpr (GATE == kGateScalar) {
        const float a0 = gbuf[2 * lane], a1 = gbuf[2 * lane + 1];
        float incl = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        float excl = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) excl = 0.f;
        const float G0 = excl + a0, G1 = incl;
        const float Gl = __shfl_sync(0xffffffffu, incl, 31);
        const float Gm = __shfl_sync(0xffffffffu, incl, 15);   // G_31
        const float G00 = __shfl_sync(0xffffffffu, G0, 0);
        gbuf[2 * lane] = G0;
        gbuf[2 * lane + 1] = G1;
        gbuf[64 + 2 * lane] = expf(G0);
        gbuf[64 + 2 * lane + 1] = expf(G1);
        gbuf[128 + 2 * lane] = expf(Gl - G0);
        gbuf[128 + 2 * lane + 1] = expf(Gl - G1);
        gbuf[256 + 2 * lane] = expf(G0 - Gm);
        gbuf[256 + 2 * lane + 1] = expf(G1 - Gm);
        gbuf[320 + 2 * lane] = expf(Gm - G0);
        gbuf[320 + 2 * lane + 1] = expf(Gm - G1);
        if (lane == 0) gbuf[384] = (G00 - Gm < 80.f && Gm - Gl < 80.f) ? 1.f : 0.f;
    } else {
        gbuf[2 * lane] = gbuf[2 * lane + 1] = 0.f;
        gbuf[64 + 2 * lane] = gbuf[64 + 2 * lane + 1] = 1.f;
        gbuf[128 + 2 * lane] = gbuf[128 + 2 * lane + 1] = 1.f;
        gbuf[256 + 2 * lane] = gbuf[256 + 2 * lane + 1] = 1.f;
        gbuf[320 + 2 * lane] = gbuf[320 + 2 * lane + 1] = 1.f;
        if (lane == 0) gbuf[384] = 1.f;
    }
}

struct PrepMaps {
    CUtensorMap q, k;
};

// Prep shared memory (bytes from a 1 KB-aligned base).
constexpr uint32_t P_OFF_KQ = 0;                          // [K_b0 | Q_b0 | K_b1 | Q_b1]
constexpr uint32_t P_OFF_AF = 32768;                      // A fp32 [64][LDF]
constexpr uint32_t P_OFF_TF = P_OFF_AF + 64 * LDF * 4;    // T fp32 [64][LDF]
constexpr uint32_t P_OFF_GATE = P_OFF_TF + 64 * LDF * 4;
constexpr uint32_t P_OFF_BAR = P_OFF_GATE + GATE_FLOATS * 4;
constexpr uint32_t P_SMEM = P_OFF_BAR + 16 + 1024;

// One CTA per chunk of the wave: everything that does not depend on the state.
template <int GATE>
__global__ void __launch_bounds__(NPR)
chunk_prep_tc_kernel(const __grid_constant__ PrepMaps maps, const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    float* Af = reinterpret_cast<float*>(sm + P_OFF_AF);
    float* Tf = reinterpret_cast<float*>(sm + P_OFF_TF);
    float* gbuf = reinterpret_cast<float*>(sm + P_OFF_GATE);
    uint64_t* bar_kq = reinterpret_cast<uint64_t*>(sm + P_OFF_BAR);
    uint64_t* bar_s = bar_kq + 1;
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, T = p.T;
    const int bh = blockIdx.x / p.nchunks, nl = blockIdx.x % p.nchunks;
    const int b = bh / H, h = bh % H;
    const int n = p.chunk0 + nl;
    uint8_t* img = p.ws + ((size_t)bh * p.cw + nl) * p.ws_chunk;
    int failed = 0;

    if (tid == 0) {
        mbar_init(bar_kq, 1);
        mbar_init(bar_s, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar_kq, 4 * 8192);
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_3d(sm + P_OFF_KQ + blk * 16384, &maps.k, bar_kq, h * D + 64 * blk, n * C, b);
            tma_load_3d(sm + P_OFF_KQ + blk * 16384 + 8192, &maps.q, bar_kq, h * D + 64 * blk, n * C, b);
        }
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 64);
        tmem_relinquish();
    }
    if (tid < 64) {
        const int t = n * C + tid;
        float gv = 0.f, bv = 0.f;
        if (t < T) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            bv = __bfloat162float(static_cast<const __nv_bfloat16*>(p.beta)[tok]);
            if constexpr (GATE == kGateScalar) gv = __bfloat162float(static_cast<const __nv_bfloat16*>(p.g)[tok]);
        }
        gbuf[tid] = gv;
        gbuf[192 + tid] = bv;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    if (warp == 0) chunk_gates<GATE>(gbuf, lane);
    if (tid == 32) {   // S = [K; Q] K^T
        if (mbar_wait(bar_kq, 0, &failed)) {
            const uint32_t st = smem_u32(sm + P_OFF_KQ);
            const uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = st + (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), id, k > 0);
            }
            mma_commit(bar_s);
        } else {
            atomicOr(p.status, kStatusTimeout);
        }
    }
    __syncthreads();
    const float* sG = gbuf;
    const float* sGam = gbuf + 64;
    const float* sFt = gbuf + 128;
    const float* sBeta = gbuf + 192;
    const float* sU = gbuf + 256;
    const float* sW = gbuf + 320;
    const bool fact = gbuf[384] != 0.f;
    if (!mbar_wait(bar_s, 0, &failed)) atomicOr(p.status, kStatusTimeout);
    __syncwarp();
    tc_fence_after();
    // A (fp32 scratch, rows 0..63) and P (bf16 image, rows 64..127)
    {
        const int q4 = warp & 3, ch = warp >> 2;
        const int L = q4 * 32 + lane;
        float sv[32];
        ld_cols<32>(tmem + ((uint32_t)(q4 * 32) << 16) + 32 * ch, sv);
        if (L < 64) {
            const int r = L;
            if (fact) {
                const float cr = sBeta[r] * sU[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * ch + e;
                    sv[e] = (i < r) ? cr * sW[i] * sv[e] : 0.f;
                }
            } else {
                const float Gr = sG[r], br = sBeta[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * ch + e;
                    sv[e] = (i < r) ? br * __expf(Gr - sG[i]) * sv[e] : 0.f;
                }
            }
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(Af + r * LDF + 32 * ch + e) =
                    make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
        } else {
            const int r = L - 64;
            if (fact) {
                const float cr = sU[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * ch + e;
                    sv[e] = (i <= r) ? cr * sW[i] * sv[e] : 0.f;
                }
            } else {
                const float Gr = sG[r];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * ch + e;
                    sv[e] = (i <= r) ? __expf(Gr - sG[i]) * sv[e] : 0.f;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_row_chunk(img + WS_P, r, 4 * ch + jj, sv + 8 * jj, 1.f);
        }
    }
    __syncthreads();
    forward_substitution(Af, Tf, tid);
    // T diag(beta) and T diag(beta e^G) as bf16 images, K-major [r][i]
    {
        const int r = tid >> 2, j0 = 2 * (tid & 3);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = j0 + jj;
            const float4 t0 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j);
            const float4 t1 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j + 4);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            float tu[8], tw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * j + e;
                tu[e] = (i <= r) ? tv[e] * sBeta[i] : 0.f;
                tw[e] = tu[e] * sGam[i];
            }
            st_row_chunk(img + WS_TU, r, j, tu, 1.f);
            st_row_chunk(img + WS_TW, r, j, tw, 1.f);
        }
    }
    if (tid < 64) {
        float* fac = reinterpret_cast<float*>(img + WS_FAC);
        fac[tid] = sGam[tid];
        fac[64 + tid] = sFt[tid];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// ------------------------------------------------------------------ per-dim
// Workspace image of one per-dimension-gated chunk: the scalar layout
// (T diag(beta) in both T slots, P, factors = e^(G_C) per key dimension),
// followed by the chain's three per-element-scaled operand tiles.
constexpr uint32_t WS_QB = WS_CHUNK;             // Q (.) e^G            [Q_b0 | Q_b1]
constexpr uint32_t WS_KG = WS_QB + 16384;        // K (.) e^G            [K_b0 | K_b1]
constexpr uint32_t WS_KT = WS_KG + 16384;        // K (.) e^(G_C - G)    [K_b0 | K_b1]
constexpr uint32_t WS_CHUNK_PD = WS_KT + 16384;

struct PrepPdMaps {
    CUtensorMap q, k, g;
};

// Per-dim prep shared memory (bytes from a 1 KB-aligned base).
constexpr int LDG = 132;                                  // fp32 row stride of G [64][128]
constexpr uint32_t D_OFF_KQ = 0;                          // [K_b0 | Q_b0 | K_b1 | Q_b1] -> scaled in place
constexpr uint32_t D_OFF_G16 = 32768;                     // g tile bf16 [g_b0 | g_b1]
constexpr uint32_t D_OFF_KB = 49152;                      // K_breve [K_b0 | K_b1], K-major rows i
constexpr uint32_t D_OFF_AF = 65536;                      // A fp32 [64][LDF]; G fp32 before it
constexpr uint32_t D_OFF_TF = D_OFF_AF + 64 * LDF * 4;    // T fp32 [64][LDF]
constexpr uint32_t D_OFF_SMALL = D_OFF_TF + 64 * LDF * 4; // beta[64], m[128], c[128], flag
constexpr uint32_t D_OFF_BAR = D_OFF_SMALL + (64 + 4 * 128 + 4) * 4;
constexpr uint32_t D_SMEM = D_OFF_BAR + 16 + 1024;
static_assert(64 * LDG * 4 <= 2 * 64 * LDF * 4, "G fits in the A/T scratch");

// One CTA per chunk of the wave (per-dimension gate).  With G the in-chunk
// cumsum of g per key dimension, m = G_31 and c = G_63 per dimension:
//   S = [K e^(G-m); Q e^(G-m)] (K e^(m-G))^T  -> A = StrictTril(beta S_kk),
//   P = Tril(S_qk); both factors and their reciprocals stay normal fp32 while
//   every dimension decays by less than e^80 in each half of the chunk, else
//   A and P are formed exactly on CUDA cores.  The chain's operands Q e^G, K e^G and K e^(G_C - G) go to the
//   workspace as shared-memory images; T diag(beta) fills both T slots (the
//   decay sits on K e^G for W).
__global__ void __launch_bounds__(NPR)
chunk_prep_pd_kernel(const __grid_constant__ PrepPdMaps maps, const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    float* Af = reinterpret_cast<float*>(sm + D_OFF_AF);
    float* Tf = reinterpret_cast<float*>(sm + D_OFF_TF);
    float* Gs = reinterpret_cast<float*>(sm + D_OFF_AF);   // G, dead before A is written
    float* sBeta = reinterpret_cast<float*>(sm + D_OFF_SMALL);
    float* sM = sBeta + 64;
    float* sC = sM + 128;
    float* sEm = sC + 128;
    float* sEcm = sEm + 128;
    int* sFlag = reinterpret_cast<int*>(sEcm + 128);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + D_OFF_BAR);
    uint64_t* bar_s = bar_ld + 1;
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, T = p.T;
    const int bh = blockIdx.x / p.nchunks, nl = blockIdx.x % p.nchunks;
    const int b = bh / H, h = bh % H;
    const int n = p.chunk0 + nl;
    uint8_t* img = p.ws + ((size_t)bh * p.cw + nl) * p.ws_chunk;
    int failed = 0;

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_s, 1);
        fence_mbar_init();
        *sFlag = 0;
        mbar_arrive_expect_tx(bar_ld, 6 * 8192);
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_3d(sm + D_OFF_KQ + blk * 16384, &maps.k, bar_ld, h * D + 64 * blk, n * C, b);
            tma_load_3d(sm + D_OFF_KQ + blk * 16384 + 8192, &maps.q, bar_ld, h * D + 64 * blk, n * C, b);
            tma_load_3d(sm + D_OFF_G16 + blk * 8192, &maps.g, bar_ld, h * D + 64 * blk, n * C, b);
        }
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 64);
        tmem_relinquish();
    }
    if (tid < 64) {
        const int t = n * C + tid;
        sBeta[tid] = (t < T) ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.beta)[((size_t)b * T + t) * H + h]) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    if (!mbar_wait(bar_ld, 0, &failed)) atomicOr(p.status, kStatusTimeout);
    __syncwarp();
    // ---- G = in-chunk cumsum of g per dimension: thread (d, half), 32 rows each
    {
        const int d = tid & 127, hh = tid >> 7;
        const uint8_t* gt = sm + D_OFF_G16 + (d >> 6) * 8192;
        float acc = 0.f;
#pragma unroll 8
        for (int r = 32 * hh; r < 32 * hh + 32; ++r) {
            acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(gt + sw128_offset(r, d & 63)));
            Gs[r * LDG + d] = acc;
        }
    }
    __syncthreads();
    {
        const int d = tid & 127, hh = tid >> 7;
        if (hh == 1) {
            const float carry = Gs[31 * LDG + d];
#pragma unroll 8
            for (int r = 32; r < 64; ++r) Gs[r * LDG + d] += carry;
        }
    }
    __syncthreads();
    if (tid < 128) {
        const float m = Gs[31 * LDG + tid], c = Gs[63 * LDG + tid];
        sM[tid] = m;
        sC[tid] = c;
        sEm[tid] = expf(m);
        sEcm[tid] = expf(c - m);
        if (Gs[tid] - m >= 80.f || m - c >= 80.f) atomicOr(sFlag, 1);
    }
    __syncthreads();
    const bool exact = *sFlag != 0;
    // ---- one pass over the tiles: Gram operands in place / K_breve, chain images
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
        const int idx = tid + NPR * it;                 // 16-byte chunk 0..1023
        const int blk = idx >> 9, r = (idx >> 3) & 63, j = idx & 7;
        const int d0 = blk * 64 + 8 * (j ^ (r & 7));    // logical columns of this chunk
        const uint32_t rowoff = (uint32_t)(r * 128 + j * 16);
        uint4 kraw = *reinterpret_cast<const uint4*>(sm + D_OFF_KQ + blk * 16384 + rowoff);
        uint4 qraw = *reinterpret_cast<const uint4*>(sm + D_OFF_KQ + blk * 16384 + 8192 + rowoff);
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kraw);
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qraw);
        uint32_t kb[4], qb[4], kr[4], qg[4], kg[4], kt[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 kf = __bfloat1622float2(k2[e]);
            const float2 qf = __bfloat1622float2(q2[e]);
            float ef[2], er[2], eg[2], et[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int d = d0 + 2 * e + u;
                const float G = Gs[r * LDG + d], m = sM[d];
                if (!exact) {
                    ef[u] = expf(G - m);
                    er[u] = expf(m - G);
                    eg[u] = sEm[d] * ef[u];     // e^G <= 1
                    et[u] = sEcm[d] * er[u];    // e^(G_C - G) <= 1
                } else {
                    ef[u] = er[u] = 0.f;
                    eg[u] = expf(G);
                    et[u] = expf(sC[d] - G);
                }
            }
            kb[e] = pack_bf16(kf.x * ef[0], kf.y * ef[1]);
            qb[e] = pack_bf16(qf.x * ef[0], qf.y * ef[1]);
            kr[e] = pack_bf16(kf.x * er[0], kf.y * er[1]);
            qg[e] = pack_bf16(qf.x * eg[0], qf.y * eg[1]);
            kg[e] = pack_bf16(kf.x * eg[0], kf.y * eg[1]);
            kt[e] = pack_bf16(kf.x * et[0], kf.y * et[1]);
        }
        const uint32_t ioff = blk * 8192 + rowoff;
        *reinterpret_cast<uint4*>(img + WS_QB + ioff) = make_uint4(qg[0], qg[1], qg[2], qg[3]);
        *reinterpret_cast<uint4*>(img + WS_KG + ioff) = make_uint4(kg[0], kg[1], kg[2], kg[3]);
        *reinterpret_cast<uint4*>(img + WS_KT + ioff) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
        if (!exact) {
            *reinterpret_cast<uint4*>(sm + D_OFF_KQ + blk * 16384 + rowoff) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
            *reinterpret_cast<uint4*>(sm + D_OFF_KQ + blk * 16384 + 8192 + rowoff) = make_uint4(qb[0], qb[1], qb[2], qb[3]);
            *reinterpret_cast<uint4*>(sm + D_OFF_KB + ioff) = make_uint4(kr[0], kr[1], kr[2], kr[3]);
        }
    }
    if (tid < 128) reinterpret_cast<float*>(img + WS_FAC)[tid] = expf(sC[tid]);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!exact) {
        if (tid == 32) {   // S = [K e^(G-m); Q e^(G-m)] (K e^(m-G))^T
            const uint32_t st = smem_u32(sm + D_OFF_KQ), kbr = smem_u32(sm + D_OFF_KB);
            const uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = st + (k >> 2) * 16384 + (k & 3) * 32;
                const uint32_t bb = kbr + (k >> 2) * 8192 + (k & 3) * 32;
                mma_bf16(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 16, 1024), id, k > 0);
            }
            mma_commit(bar_s);
        }
        if (!mbar_wait(bar_s, 0, &failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
        tc_fence_after();
        __syncthreads();   // G (aliased with A) is dead from here on
        const int q4 = warp & 3, ch = warp >> 2;
        const int L = q4 * 32 + lane;
        float sv[32];
        ld_cols<32>(tmem + ((uint32_t)(q4 * 32) << 16) + 32 * ch, sv);
        if (L < 64) {
            const int r = L;
            const float br = sBeta[r];
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[e] = (32 * ch + e < r) ? br * sv[e] : 0.f;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(Af + r * LDF + 32 * ch + e) = make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
        } else {
            const int r = L - 64;
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[e] = (32 * ch + e <= r) ? sv[e] : 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_row_chunk(img + WS_P, r, 4 * ch + jj, sv + 8 * jj, 1.f);
        }
    } else {
        // exact A and P: sum_d k_rd k_id e^(G_rd - G_id) with every exponent <= 0;
        // A goes to registers first since it shares space with G
        const int q4 = warp & 3, ch = warp >> 2;
        const int L = q4 * 32 + lane;
        const int r = L & 63;
        const bool isq = L >= 64;
        const uint8_t* rowt = sm + D_OFF_KQ + (isq ? 8192 : 0);
        float sv[32];
#pragma unroll 1
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * ch + e;
            float acc = 0.f;
            if (isq ? (i <= r) : (i < r)) {
#pragma unroll 4
                for (int d = 0; d < D; ++d) {
                    const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                        rowt + (d >> 6) * 16384 + sw128_offset(r, d & 63)));
                    const float kk = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                        sm + D_OFF_KQ + (d >> 6) * 16384 + sw128_offset(i, d & 63)));
                    acc = fmaf(x * kk, expf(Gs[r * LDG + d] - Gs[i * LDG + d]), acc);
                }
            }
            sv[e] = isq ? acc : sBeta[r] * acc;
        }
        __syncthreads();   // G (aliased with A) is dead from here on
        if (!isq) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(Af + r * LDF + 32 * ch + e) = make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
        } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_row_chunk(img + WS_P, r, 4 * ch + jj, sv + 8 * jj, 1.f);
        }
    }
    __syncthreads();
    forward_substitution(Af, Tf, tid);
    {
        const int r = tid >> 2, j0 = 2 * (tid & 3);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = j0 + jj;
            const float4 t0 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j);
            const float4 t1 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j + 4);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            float tu[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * j + e;
                tu[e] = (i <= r) ? tv[e] * sBeta[i] : 0.f;
            }
            st_row_chunk(img + WS_TU, r, j, tu, 1.f);
            st_row_chunk(img + WS_TW, r, j, tu, 1.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// Chain kernel shared memory (bytes from a 1 KB-aligned base).
constexpr uint32_t KQ_STAGE = 32768;   // [K_b0 | Q_b0 | K_b1 | Q_b1], 8 KB each, K-major
constexpr uint32_t OFF_KQ = 0;         // 2 stages
constexpr uint32_t OFF_V = 65536;      // 2 buffers of [V_b0 | V_b1]
constexpr uint32_t OFF_TU = 98304;     // T diag(beta)          } [T_u; Z] and
constexpr uint32_t OFF_Z = 106496;     // zero block            } [Z; T_w] are
constexpr uint32_t OFF_TW = 114688;    // T diag(beta e^G)      } 128-row stacks
constexpr uint32_t OFF_Z2 = 122880;    // zero block            } [Z2; P]
constexpr uint32_t OFF_P = 131072;     // P, K-major [64 r][64 i]
constexpr uint32_t OFF_WQ = 139264;    // [-W_b0 | Qbar_b0 | -W_b1 | Qbar_b1], K-major
constexpr uint32_t OFF_HB = 172032;    // h (bf16) MN-major [d][64 v] x 2; after the
constexpr uint32_t OFF_DL = 172032;    //   c-MMA: D [i][64 v] x 2 (first 16 KB)
constexpr uint32_t OFF_KT = 204800;    // K~ = diag(e^(G_C - G_i)) K, [K~_b0 | K~_b1]
constexpr uint32_t OFF_FAC = 221184;   // 2 x {e^G [64], e^(G_C - G) [64]}
constexpr uint32_t OFF_BAR = OFF_FAC + 2 * 128 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 32 * 8 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr int NT = 288;          // 9 warps
constexpr int NCH = 128;         // chain threads (warps 0-3)
constexpr int NST = 128;         // stager threads (warps 4-7)

// TMEM columns (512 allocated).
constexpr uint32_t TM_H = 0;      // state, lanes d, 128 columns v (fp32)
constexpr uint32_t TM_X0 = 128;   // X for even chunks, lanes r / 64 + r, 128 columns v
constexpr uint32_t TM_X1 = 256;   // X for odd chunks
constexpr uint32_t TM_W = 384;    // [0; W], lanes 64..127, 128 columns d

enum Bar {
    B_KQ0, B_KQ1, B_VFULL, B_TFULL, B_PFULL, B_FFULL0, B_FFULL1, B_WUDONE, B_CDONE, B_DDONE,
    B_WQREADY, B_HBREADY, B_DREADY, B_XFREE, B_QFULL, B_FINAL, B_COUNT
};

struct TcMaps {
    CUtensorMap q, k, v;
};

__global__ void __launch_bounds__(NT, 1)
chunk_fwd_tc_kernel(const __grid_constant__ TcMaps maps, const ChunkParams p, int gated, int perdim) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, T = p.T;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int NC = p.nchunks;              // local chunk nl = 0..NC-1 is chunk p.chunk0 + nl
    const uint8_t* wsh = p.ws + (size_t)bh * p.cw * p.ws_chunk;
    int failed = 0;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        prefetch_tmap(&maps.q);
        prefetch_tmap(&maps.k);
        prefetch_tmap(&maps.v);
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    for (int i = tid; i < 1024; i += NT) {   // the two zero blocks
        const uint32_t off = (i < 512) ? OFF_Z + 16 * i : OFF_Z2 + 16 * (i - 512);
        *reinterpret_cast<uint4*>(sm + off) = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;

    auto fac_buf = [&](int nl) { return reinterpret_cast<float*>(sm + OFF_FAC) + (nl & 1) * 128; };
    auto wait = [&](int bar, uint32_t parity) {
        if (!mbar_wait(&bars[bar], parity, &failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    };
    auto load_kq = [&](int nl) {
        const int s = nl & 1, n = p.chunk0 + nl;
        mbar_arrive_expect_tx(&bars[B_KQ0 + s], 4 * 8192);
        uint8_t* st = sm + OFF_KQ + s * KQ_STAGE;
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_3d(st + blk * 16384, &maps.k, &bars[B_KQ0 + s], h * D + 64 * blk, n * C, b);
            tma_load_3d(st + blk * 16384 + 8192, &maps.q, &bars[B_KQ0 + s], h * D + 64 * blk, n * C, b);
        }
    };
    auto load_v = [&](int nl) {
        const int n = p.chunk0 + nl;
        mbar_arrive_expect_tx(&bars[B_VFULL], 2 * 8192);
        for (int blk = 0; blk < 2; ++blk)
            tma_load_3d(sm + OFF_V + (nl & 1) * 16384 + blk * 8192, &maps.v, &bars[B_VFULL],
                        h * D + 64 * blk, n * C, b);
    };

    if (warp == 8) {
        // =========================== control: TMA for the first tiles and V, every MMA
        const bool leader = lane == 0;   // issues only while no wait has failed
        if (leader && !perdim) {
            fence_async_smem();
            load_kq(0);
            if (NC > 1) load_kq(1);
        }
        // W and U of chunk nl: operands loaded, TMEM free (for nl >= 2 the output
        // of chunk nl - 2 has been read out of X[nl & 1])
        auto issue_wu = [&](int nl) {
            const int s = nl & 1;
            const uint32_t st = sb + OFF_KQ + s * KQ_STAGE;
            const uint32_t tX = tmem + (s ? TM_X1 : TM_X0);
            wait(B_TFULL, nl & 1);
            wait(B_VFULL, nl & 1);
            if (!perdim) wait(B_KQ0 + s, (nl >> 1) & 1);
            if (nl >= 2) wait(B_XFREE, (nl - 2) & 1);
            tc_fence_after();
            if (leader && !failed) {
                const uint32_t idw = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // [0; W] = [Z; T_w] K
                    mma_bf16(tmem + TM_W, sdesc_sw128(sb + OFF_Z + k * 32, 16, 1024),
                             sdesc_sw128(st + k * 2048, 16384, 1024), idw, k > 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // X = [T_u; Z] V
                    mma_bf16(tX, sdesc_sw128(sb + OFF_TU + k * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_V + s * 16384 + k * 2048, 8192, 1024), idw, k > 0);
                mma_commit(&bars[B_WUDONE]);
            }
        };
        if (NC > 0) issue_wu(0);
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            const uint32_t tX = tmem + (s ? TM_X1 : TM_X0);
            wait(B_WQREADY, nl & 1);
            wait(B_HBREADY, nl & 1);
            tc_fence_after();
            if (leader && !failed) {
                const uint32_t idc = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
                for (int k = 0; k < 8; ++k)   // X += [-W; Q_bar] h
                    mma_bf16(tX, sdesc_sw128(sb + OFF_WQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_HB + k * 2048, 16384, 1024), idc, true);
                mma_commit(&bars[B_CDONE]);
            }
            // the next chunk's W / U run while the chain turns D of this one
            if (nl + 1 < NC) issue_wu(nl + 1);
            wait(B_DREADY, nl & 1);
            wait(B_PFULL, nl & 1);
            tc_fence_after();
            if (leader && !failed) {
                const uint32_t id2 = idesc_bf16_f32(128, 128, true, true);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // state += K~^T D
                    mma_bf16(tmem + TM_H, sdesc_sw128(sb + OFF_KT + k * 2048, 8192, 1024),
                             sdesc_sw128(sb + OFF_DL + k * 2048, 8192, 1024), id2, true);
                const uint32_t id1 = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
                for (int k = 0; k < 4; ++k)   // X += [Z2; P] D
                    mma_bf16(tX, sdesc_sw128(sb + OFF_Z2 + k * 32, 16, 1024),
                             sdesc_sw128(sb + OFF_DL + k * 2048, 8192, 1024), id1, true);
                mma_commit(&bars[B_DDONE]);
            }
        }
        // nothing issued by this warp may still run when TMEM is released
        if (leader) mma_commit(&bars[B_FINAL]);
        int final_failed = 0;
        if (!mbar_wait(&bars[B_FINAL], 0, &final_failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    } else if (warp >= 4) {
        // =========================== stager: prep images in, -W and Q_bar operands
        const int st_id = tid - NCH;                // 0..127
        const int L = (warp & 3) * 32 + lane;       // TMEM lane of this thread
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            const uint8_t* img = wsh + (size_t)nl * p.ws_chunk;
            if (st_id == 0) {   // W/U of chunk nl-1 are done with T_u / T_w, and the chain is
                                // done with the factors of chunk nl-2 (both waited below)
                mbar_arrive_expect_tx(&bars[B_TFULL], perdim ? 4 * 8192 : 2 * 8192);
                bulk_load(sm + OFF_TU, img + WS_TU, 8192, &bars[B_TFULL]);
                bulk_load(sm + OFF_TW, img + WS_TW, 8192, &bars[B_TFULL]);
                if (perdim) {   // K e^G into the K slots of stage nl & 1 (W of chunk nl-2 is done)
                    uint8_t* stg = sm + OFF_KQ + s * KQ_STAGE;
                    bulk_load(stg, img + WS_KG, 8192, &bars[B_TFULL]);
                    bulk_load(stg + 16384, img + WS_KG + 8192, 8192, &bars[B_TFULL]);
                }
                mbar_arrive_expect_tx(&bars[B_FFULL0 + s], 512);
                bulk_load(fac_buf(nl), img + WS_FAC, 512, &bars[B_FFULL0 + s]);
                fence_async_smem();
                load_v(nl);   // V buffer nl & 1: U of chunk nl-2 is long done
            }
            // Q_bar = diag(e^G) Q into the Q rows of WQ (same swizzled layout) once the
            // c-product of chunk nl-1 is done with WQ, and K~ = diag(e^(G_C - G)) K
            // once the state update of chunk nl-1 is done with K~
            if (nl > 0) wait(B_CDONE, (nl - 1) & 1);
            wait(B_FFULL0 + s, (nl >> 1) & 1);
            if (!perdim) wait(B_KQ0 + s, (nl >> 1) & 1);
            const float* fac = fac_buf(nl);
            const uint8_t* stage = sm + OFF_KQ + s * KQ_STAGE;
            auto scale_rows = [&](uint32_t src_off, uint8_t* dst, const float* rowf) {
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int idx = st_id + NST * it;          // 16-byte chunk 0..1023
                    const int blk = idx >> 9, r = (idx >> 3) & 63, j = idx & 7;
                    uint4 raw = *reinterpret_cast<const uint4*>(stage + blk * 16384 + src_off + r * 128 + j * 16);
                    const float gmul = rowf[r];
                    __nv_bfloat162* e2 = reinterpret_cast<__nv_bfloat162*>(&raw);
                    uint4 outv;
                    uint32_t* o32 = reinterpret_cast<uint32_t*>(&outv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(e2[e]);
                        o32[e] = pack_bf16(f.x * gmul, f.y * gmul);
                    }
                    *reinterpret_cast<uint4*>(dst + blk * (dst == sm + OFF_KT ? 8192 : 16384) + r * 128 + j * 16) = outv;
                }
            };
            if (!perdim) {
                scale_rows(8192, sm + OFF_WQ + 8192, fac);   // Q rows -> Q_bar rows of WQ
            } else if (st_id == 0) {                         // Q e^G image -> Q_bar rows of WQ
                mbar_arrive_expect_tx(&bars[B_QFULL], 2 * 8192);
                bulk_load(sm + OFF_WQ + 8192, img + WS_QB, 8192, &bars[B_QFULL]);
                bulk_load(sm + OFF_WQ + 8192 + 16384, img + WS_QB + 8192, 8192, &bars[B_QFULL]);
            }
            // -W (TMEM lanes 64..127, warps 6-7) -> the W rows of WQ
            wait(B_WUDONE, nl & 1);
            tc_fence_after();
            if (L >= 64) {
                const int r = L - 64;
                float wv[128];
                ld_cols<128>(tmem + TM_W + lane_off, wv);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    st_row_chunk(sm + OFF_WQ + (j >> 3) * 16384, r, j & 7, wv + 8 * j, -1.f);
            }
            if (perdim) wait(B_QFULL, nl & 1);
            fence_async_smem();
            tc_fence_before();
            named_bar(3, NST);
            if (st_id == 0) mbar_arrive(&bars[B_WQREADY]);
            // P and K~ of chunk nl once the d-products of chunk nl-1 are done with them
            if (nl > 0) wait(B_DDONE, (nl - 1) & 1);
            if (!perdim) {
                scale_rows(0, sm + OFF_KT, fac + 64);      // K rows -> K~
                fence_async_smem();
                named_bar(3, NST);
            }
            if (st_id == 0) {
                mbar_arrive_expect_tx(&bars[B_PFULL], perdim ? 3 * 8192 : 8192);
                bulk_load(sm + OFF_P, img + WS_P, 8192, &bars[B_PFULL]);
                if (perdim) bulk_load(sm + OFF_KT, img + WS_KT, 16384, &bars[B_PFULL]);
            }
        }
    } else {
        // =========================== chain: state, D, output
        {
            const float* s0 = p.s0 ? p.s0 + ((size_t)bh * D + tid) * D : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = s0 ? s0[c0 + j] : 0.f;
                tmem_st16(tmem + TM_H + lane_off + c0, v);
            }
            tmem_wait_st();
        }
        auto out_epilogue = [&](int ml) {   // chunk ml's O, warps 2-3 (TMEM lanes 64..127)
            const int r = tid - 64, t0 = (p.chunk0 + ml) * C;
            const int nval = min(C, T - t0);
            const uint32_t tX = tmem + ((ml & 1) ? TM_X1 : TM_X0);
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) + (((size_t)b * T + t0 + r) * H + h) * D;
            float ov[128];
            ld_cols<128>(tX + lane_off, ov);
            if (r < nval) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    uint4 w;
                    w.x = pack_bf16(ov[8 * j + 0], ov[8 * j + 1]);
                    w.y = pack_bf16(ov[8 * j + 2], ov[8 * j + 3]);
                    w.z = pack_bf16(ov[8 * j + 4], ov[8 * j + 5]);
                    w.w = pack_bf16(ov[8 * j + 6], ov[8 * j + 7]);
                    *reinterpret_cast<uint4*>(orow + 8 * j) = w;
                }
            }
        };
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            if (nl > 0) {
                wait(B_DDONE, (nl - 1) & 1);
                tc_fence_after();
                if (tid == 0 && nl + 1 < NC && !perdim) {
                    fence_async_smem();
                    load_kq(nl + 1);
                }
            }
            // state -> bf16 operand h (MN-major [d][64 v] x 2), row d = tid
            {
                float hv[128];
                ld_cols<128>(tmem + TM_H + lane_off, hv);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    st_row_chunk(sm + OFF_HB + (j >> 3) * 16384, tid, j & 7, hv + 8 * j, 1.f);
            }
            fence_async_smem();
            named_bar(1, NCH);
            if (tid == 0) mbar_arrive(&bars[B_HBREADY]);
            // state *= e^(G_C) (before the state update of this chunk)
            wait(B_FFULL0 + s, (nl >> 1) & 1);
            const float* fac = fac_buf(nl);
            if (gated) {
                const float gam = perdim ? fac[tid] : fac[63];
                float hv[128];
                ld_cols<128>(tmem + TM_H + lane_off, hv);
#pragma unroll
                for (int e = 0; e < 128; ++e) hv[e] *= gam;
                st_cols<128>(tmem + TM_H + lane_off, hv);
                tmem_wait_st();
            }
            tc_fence_before();
            named_bar(1, NCH);
            if (warp >= 2) {
                if (nl > 0) {
                    out_epilogue(nl - 1);
                    tc_fence_before();
                    named_bar(4, 64);
                    if (tid == 64) mbar_arrive(&bars[B_XFREE]);   // X[(nl - 1) & 1] is free
                }
            } else {
                wait(B_CDONE, nl & 1);
                tc_fence_after();
                const uint32_t tX = tmem + (s ? TM_X1 : TM_X0);
                float dv[128];
                ld_cols<128>(tX + lane_off, dv);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    st_row_chunk(sm + OFF_DL + (j >> 3) * 8192, tid, j & 7, dv + 8 * j, 1.f);
            }
            fence_async_smem();
            tc_fence_before();
            named_bar(1, NCH);
            if (tid == 0) mbar_arrive(&bars[B_DREADY]);
        }
        if (NC > 0) {
            wait(B_DDONE, (NC - 1) & 1);
            tc_fence_after();
            if (warp >= 2) out_epilogue(NC - 1);
            if (!failed && p.s_out) {
                float* dst = p.s_out + ((size_t)bh * D + tid) * D;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float hv[64];
                    ld_cols<64>(tmem + TM_H + lane_off + 64 * half, hv);
#pragma unroll
                    for (int e = 0; e < 64; e += 4)
                        *reinterpret_cast<float4*>(dst + 64 * half + e) = make_float4(hv[e], hv[e + 1], hv[e + 2], hv[e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

bool make_maps(const ChunkParams& p, TcMaps* m) {
    const uint64_t dims[3] = {(uint64_t)p.H * D, (uint64_t)p.T, (uint64_t)p.B};
    const uint64_t strides[2] = {(uint64_t)p.H * D * 2, (uint64_t)p.T * p.H * D * 2};
    const uint32_t box[3] = {64, 64, 1};
    return make_tmap_bf16(&m->q, p.q, 3, dims, strides, box) &&
           make_tmap_bf16(&m->k, p.k, 3, dims, strides, box) &&
           make_tmap_bf16(&m->v, p.v, 3, dims, strides, box);
}

// Chunk slots per (batch, head) of one wave: as many as keep the wave's
// workspace near WAVE_BYTES (L2-resident), at least 4.
int wave_chunks(int nbh, int NC, uint32_t image_bytes) {
    long long cw = (long long)(WAVE_BYTES / ((size_t)nbh * image_bytes));
    if (cw < 4) cw = 4;
    if (cw > NC) cw = NC;
    return (int)(cw < 1 ? 1 : cw);
}

}  // namespace

bool chunk_fwd_tc_supported(int Dk, int Dv, int gate) {
    return Dk == D && Dv == D && (gate == kGateNone || gate == kGateScalar || gate == kGatePerDim);
}

namespace {
uint32_t image_bytes(int gate) { return gate == kGatePerDim ? WS_CHUNK_PD : WS_CHUNK; }
}  // namespace

size_t chunk_fwd_tc_workspace_bytes(int B, int T, int H, int gate) {
    const int NC = (T + C - 1) / C;
    if (NC == 0 || B == 0 || H == 0) return 0;
    const int nbh = B * H;
    const int cw = wave_chunks(nbh, NC, image_bytes(gate));
    const int nw = (NC + cw - 1) / cw;
    size_t bytes = (size_t)nbh * cw * image_bytes(gate);
    if (nw > 1) bytes += (size_t)nbh * D * D * sizeof(float);   // state between waves
    return bytes;
}

cudaError_t launch_chunk_fwd_tc(const ChunkParams& p0, int gate, cudaStream_t s, int* launches) {
    *launches = 0;
    TcMaps maps;
    if (!make_maps(p0, &maps)) return cudaErrorInvalidValue;
    const bool perdim = gate == kGatePerDim;
    PrepMaps pmaps;
    pmaps.q = maps.q;
    pmaps.k = maps.k;
    PrepPdMaps dmaps;
    dmaps.q = maps.q;
    dmaps.k = maps.k;
    if (perdim) {
        const uint64_t dims[3] = {(uint64_t)p0.H * D, (uint64_t)p0.T, (uint64_t)p0.B};
        const uint64_t strides[2] = {(uint64_t)p0.H * D * 2, (uint64_t)p0.T * p0.H * D * 2};
        const uint32_t box[3] = {64, 64, 1};
        if (!make_tmap_bf16(&dmaps.g, p0.g, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    auto prep = gate == kGateScalar ? chunk_prep_tc_kernel<kGateScalar> : chunk_prep_tc_kernel<kGateNone>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_prep_pd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)D_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int NC = (p0.T + C - 1) / C;
    const int nbh = p0.B * p0.H;
    const uint32_t img = image_bytes(gate);
    const int cw = wave_chunks(nbh, NC, img);
    const int nw = (NC + cw - 1) / cw;
    float* carry = nw > 1 ? reinterpret_cast<float*>(p0.ws + (size_t)nbh * cw * img) : nullptr;
    for (int w = 0; w < nw; ++w) {
        ChunkParams p = p0;
        p.cw = cw;
        p.ws_chunk = (int)img;
        p.chunk0 = w * cw;
        p.nchunks = (w + 1 < nw) ? cw : NC - w * cw;
        p.s0 = (w == 0) ? p0.s0 : carry;
        p.s_out = (w + 1 == nw) ? p0.s_out : carry;
        if (perdim)
            chunk_prep_pd_kernel<<<(unsigned)(nbh * p.nchunks), NPR, D_SMEM, s>>>(dmaps, p);
        else
            prep<<<(unsigned)(nbh * p.nchunks), NPR, P_SMEM, s>>>(pmaps, p);
        ++*launches;
        chunk_fwd_tc_kernel<<<(unsigned)nbh, NT, SMEM_BYTES, s>>>(maps, p, gate != kGateNone ? 1 : 0,
                                                                  perdim ? 1 : 0);
        ++*launches;
    }
    return cudaGetLastError();
}

}  // namespace gdn
