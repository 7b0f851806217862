// chunk_fwd_tc.cu -- chunkwise gated delta rule on the sm_100a tensor cores
// (bf16 operands, fp32 accumulation in TMEM, fp32 state), d_k = d_v = 128.
//
// The chunkwise algorithm of "Moonshot AI's New Attention Architecture: Key
// Innovations Explained" (sec. 3, state recurrence and causal output) with the
// UT/WY transform of "OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention" (sec. 2.1, chunk Gram matrix + WY).
// Per chunk of C = 64 tokens, h the entering state M = S^T [d_k][d_v], G the
// in-chunk log-decay cumsum (per token, or per token and key dimension):
//   A  = StrictTril(diag(beta) (K e^G)(K e^-G)^T),  P = Tril((Q e^G)(K e^-G)^T)
//   T  = (I + A)^-1                               (blocked forward substitution)
//   W  = T diag(beta) (K e^G),  U = T diag(beta) V,  K~ = K e^(G_C - G)
//   D  = U - W h,  O = (Q e^G) h + P D,  h' = Diag(e^(G_C)) h + K~^T D.
// Substituting D, each chunk is an affine map of the entering state:
//   h' = Diag(gamma) h + Phi h + K~^T U,    Phi = -K~^T W,  gamma = e^(G_C)
//   O  = Qp h + P U,                        Qp  = Q e^G - P W
// Phi, K~, U, Qp, P and gamma depend on the chunk's inputs only, so they are
// formed for every chunk at once, and only the products with h remain on the
// serial path.  The decay stays an fp32 multiply of the fp32 state (a bf16
// gamma - 1 folded into Phi would leave 2^-9 |h| per chunk behind, large
// against a strongly decayed h').
//
// Two kernels per wave of chunks:
//   chunk_prep_kernel   one CTA per (batch, head, chunk), fully parallel: the
//                       gates, S = [K;Q]K^T, A and P, T, the WY factors as
//                       W^T = K^T T^T and U^T = V^T T^T, then K~^T W and
//                       W^T P^T; writes the chunk's step image ([Phi ; Qp],
//                       [K~^T ; P], U^T in bf16, gamma in fp32) to the
//                       workspace by bulk copies, laid out exactly as the chain
//                       kernel's shared-memory operands;
//   chunk_chain_kernel  one CTA per (batch, head), the serial state chain on
//                       the transposed state h^T [v][d]: per chunk two MMAs of
//                       N = 192 into one TMEM accumulator, D = U^T [K~ | P^T]
//                       (off the serial path) and D += h^T [Phi^T | Qp^T] with
//                       the bf16 copy of h^T in TMEM as the A operand; columns
//                       0..127 of D feed the state pass h'^T = h^T Diag(gamma)
//                       + X^T in fp32 registers, columns 128..191 are O^T
//                       (value rows in the TMEM lanes), written by TMA stores.
// A wave's prep overlaps the previous wave's chain (programmatic dependent
// launch); two image buffers alternate between waves.
// Every mbarrier wait is bounded; a wait that gives up sets the library status
// word and the kernel winds down without further waits.
#include <string.h>

#include <algorithm>

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

// Step image of one chunk (bytes).  Tiles of bf16 rows of 64 elements with the
// 128-byte swizzle.  The chain runs two products per chunk, each with one
// K-major B operand of 192 rows (N = 192):
//   D  = U^T [K~ | P^T]     B = [K~^T ; P]  rows d (128) then r (64), K = i
//   D += h^T [Phi^T | Qp^T] B = [Phi ; Qp]  rows d' (128) then r (64), K = d
// so that columns 0..127 of D are the state update X^T and 128..191 the
// output O^T of the chunk.
constexpr uint32_t IMG_PQ = 0;         // [Phi ; Qp]: two K-blocks (d 0..63, 64..127) of
                                       //   [192][64] = 24 KB: Phi rows 0..127, Qp rows 128..191
constexpr uint32_t IMG_KP = 49152;     // [K~^T ; P]: [192][64] (K~^T rows d, then P rows r)
constexpr uint32_t IMG_UT = 73728;     // U^T  [128 v][64 i]     (K-major A)
constexpr uint32_t IMG_GAM = 90112;    // gamma fp32 [128]
constexpr uint32_t IMG_BYTES = 90624;
constexpr uint32_t PQ_BLK = 24576;     // one K-block of [Phi ; Qp]
static_assert(IMG_BYTES == kImgBytes && IMG_PQ == kImgPQ && PQ_BLK == kImgPQBlock &&
              IMG_GAM == kImgGam, "image layout the backward reads");
constexpr size_t WAVE_BYTES = size_t(160) << 20;  // cap of one wave's image buffer
constexpr int PREP_SLOTS = 2 * 148;                // prep CTAs resident at once on a B200

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&t);
}

// Chunk j (8 elements) of row `row` of a [rows][64] swizzled bf16 tile.
__device__ __forceinline__ void st_row_chunk(uint8_t* tile, int row, int j, const float* v,
                                             float scale) {
    uint4 w;
    w.x = pack_bf16(v[0] * scale, v[1] * scale);
    w.y = pack_bf16(v[2] * scale, v[3] * scale);
    w.z = pack_bf16(v[4] * scale, v[5] * scale);
    w.w = pack_bf16(v[6] * scale, v[7] * scale);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, 8 * j)) = w;
}

__device__ __forceinline__ float ld_bf16(const uint8_t* tile, int row, int col) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + sw128_offset(row, col)));
}

// Programmatic dependent launch: let the next kernel in the stream start now /
// wait until the previous one has completed and its writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Drop `bytes` (a multiple of 128) of L2 lines at p without writing them back:
// for data that is dead once read (a step image after its chain has loaded it),
// so the L2 does not spend DRAM bandwidth evicting it.  One warp, lanes split
// the lines.
__device__ __forceinline__ void l2_discard(const void* p, uint32_t bytes, int lane) {
    if (reinterpret_cast<uintptr_t>(p) & 127u) return;   // whole lines only (a workspace need
                                                          // only be 16-byte aligned)
    const char* c = static_cast<const char*>(p);
    for (uint32_t off = 128u * lane; off < bytes; off += 128u * 32u)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(c + off) : "memory");
}


template <int N>
__device__ __forceinline__ void ld_cols(uint32_t addr, float (&v)[N]) {
    static_assert(N % 16 == 0, "");
    if constexpr (N % 64 == 0) {
#pragma unroll
        for (int j = 0; j < N / 64; ++j)
            tmem_ld64(addr + 64 * j, *reinterpret_cast<float(*)[64]>(v + 64 * j));
    } else if constexpr (N % 32 == 0) {
#pragma unroll
        for (int j = 0; j < N / 32; ++j)
            tmem_ld32(addr + 32 * j, *reinterpret_cast<float(*)[32]>(v + 32 * j));
    } else {
#pragma unroll
        for (int j = 0; j < N / 16; ++j)
            tmem_ld16(addr + 16 * j, *reinterpret_cast<float(*)[16]>(v + 16 * j));
    }
    tmem_wait_ld();
    reg_fence(v);
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
// substitution on CUDA cores, one column per thread (threads 64.. run `idle`
// meanwhile); (2) 16 -> 32:
// T_10 = -T_11 (A_10 T_00) for the two diagonal 32 x 32 blocks; (3) 32 -> 64:
// the same with 32 x 32 blocks.  The block products run as warp MMAs on tf32
// operands with fp32 accumulation (T is rounded to bf16 right after, so the
// tf32 operand rounding stays well below that); the inner product X goes
// through the strictly upper part of Tm, which T never uses.
template <typename Idle>
__device__ __forceinline__ void forward_substitution(const float* A, float* Tm, int pt, Idle&& idle) {
    const int lane = pt & 31, w = pt >> 5;
    if (pt >= 64) idle(pt - 64);   // other work while two warps take the diagonal blocks
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
    CUtensorMap q, k, v, g;   // g only for the per-dimension gate
    CUtensorMap kw;           // the write key (preconditioned delta rule) only
};

// Prep shared memory (bytes from a 1 KB-aligned base); 111 KB for either
// gate, so two CTAs share an SM.
constexpr uint32_t P_KQ = 0;                 // [K_b0 | Q_b0 | K_b1 | Q_b1] (TMA);
                                             // per-dimension gate: K e^(G-c), Q e^(G-c) over K, Q
constexpr uint32_t P_V = 32768;              // [V_b0 | V_b1] (TMA)
constexpr uint32_t P_AF = 49152;             // A fp32 [64][LDF]; later [W^T; U^T] bf16 [256][64]
constexpr uint32_t P_TF = P_AF + 64 * LDF * 4;   // T fp32 [64][LDF]
constexpr uint32_t P_WUT = P_AF;
constexpr uint32_t P_TU = P_AF;              // T diag(beta) bf16 [64 r][64 i] over the dead A scratch
constexpr uint32_t P_TW = P_AF + 8192;       // T diag(beta e^G) (scalar gate)
constexpr uint32_t P_KT = 86016;             // K~^T [128 d][64 i] (K~ = K e^(G_C - G)); the
                                             // per-dimension gate's g tile lands there first
constexpr uint32_t P_P = 102400;             // P bf16 [64 r][64 i]
constexpr uint32_t P_GATE = 110592;          // scalar: G, e^G, e^(G_C-G), beta, u, w, flag;
                                             // per-dimension: beta, gamma_d, e^(ref_d)  (512 floats)
constexpr uint32_t P_BAR = P_GATE + 8 * 64 * 4;
constexpr uint32_t P_SMEM = P_BAR + 64 + 1024;
constexpr uint32_t PD_KT = P_KT;             // per-dimension gate: g bf16 (TMA), then K~
// staging of the step image for its bulk stores (buffers dead by then)
constexpr uint32_t S_PHI = 32768;            // over V and the W^T rows
constexpr uint32_t S_QPT = P_KT;             // Qp [64 r][128 d] as two [64][64] blocks, over
                                             // K~^T: dead once the K~^T W product is done and
                                             // K~^T's image store has read it
constexpr int LDG = 132;                     // fp32 row stride of G [64][128] (exact fallback; aliases A / T)
static_assert(P_TF + 64 * LDF * 4 <= P_KT, "A / T scratch");
static_assert(P_WUT + 32768 <= P_KT, "[W^T; U^T] tile");
static_assert(P_TW + 8192 <= P_TF && P_KT + 16384 <= P_P, "T_u / T_w over A, K~ tile");
static_assert(S_PHI + 32768 <= P_WUT + 16384 && S_QPT + 16384 <= P_P, "staging clear of the U^T rows and P");
static_assert(P_P == P_KT + 16384, "P right after K~^T: rows 64..127 of the A operand of P W");
static_assert(64 * LDG * 4 <= 2 * 64 * LDF * 4, "G fits in the A / T scratch");
static_assert(2 * (P_SMEM + 1024) <= 233472, "two prep CTAs per SM");

// TMEM columns of the prep kernel (256 allocated: two CTAs per SM).
constexpr uint32_t TM_S = 0;       // [K;Q] K^T, 64 columns
constexpr uint32_t TM_WT = 64;     // W^T, lanes d, 64 columns r
constexpr uint32_t TM_UT = 128;    // U^T, lanes v, 64 columns r
constexpr uint32_t TM_FP = 0;      // K~^T W, lanes d, 128 columns d'   (after S, W^T, U^T are read)
constexpr uint32_t TM_PW = 128;    // P W, lanes 64 + r, 128 columns d (lanes 0..63 unused)

// One CTA per (batch, head, chunk) of the wave: every state-independent part
// of the chunk, written to the workspace as the chunk's step image.
// WK: a separate write key kw (the preconditioned delta rule of "OSDN ...",
// sec. 2.1): the read key k stays in the A side of the Gram matrix and in W;
// kw replaces k as the B side of the Gram matrix and of the intra-chunk scores
// and in K~ (state update, Phi).  The kw tile occupies the V slot until its
// last reader is done; V is loaded there afterwards, ahead of the U^T product.
template <int GATE, bool WK>
__global__ void __launch_bounds__(NPR, 2)
chunk_prep_kernel(const __grid_constant__ PrepMaps maps, const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    float* Af = reinterpret_cast<float*>(sm + P_AF);
    float* Tf = reinterpret_cast<float*>(sm + P_TF);
    float* gbuf = reinterpret_cast<float*>(sm + P_GATE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P_BAR);   // kq, s, wu, f, v
    __shared__ uint32_t s_tmem;
    constexpr bool PD = GATE == kGatePerDim;
    // the g tile and the write key feed the first step of an item: their loads
    // (and V's) are issued at the end of the previous item; otherwise V alone,
    // needed only by the U^T product, is issued after the item's first barrier
    constexpr bool EARLY = PD || WK;

    // The grid's last block only waits for the kernel before it (the previous
    // wave's chain): this grid then completes after that chain, so the chain of
    // this wave -- and the prep of the next wave, which reuses the previous
    // wave's image buffer -- start only once it is done.  The other blocks write
    // this wave's buffer, which nothing in flight reads.
    if (blockIdx.x == gridDim.x - 1) {
        pdl_wait();
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, T = p.T;
    const int nitems = p.B * p.H * p.nchunks;
    const uint64_t pol_in = l2_evict_first();    // inputs: read once
    const uint64_t pol_img = l2_evict_last();    // step images: read back by the chain soon
    const uint32_t sb = smem_u32(sm);
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int failed = 0;
    bool rest_issued = false;   // thread 0: the next item's g / write key / V loads are out
    uint32_t ph = 0;   // phase of every barrier: each completes once per item
    auto wait = [&](int i, uint32_t parity) {
        if (!mbar_wait(&bars[i], parity, &failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    };

    float* sBeta = gbuf + 192;
    // per-dimension gate
    float* Gs = reinterpret_cast<float*>(sm + P_AF);   // exact fallback: G [64][LDG], dead before A is written
    float* sGamD = gbuf + 256;                         // gamma_d = e^(c_d)
    float* sRef = gbuf + 384;                          // e^(c_d); 1 in the exact fallback

    // Items are claimed one ahead, by one thread, which also stores the item's
    // (sequence, head, chunk, sequence * H + head) for every thread to read, so
    // that no thread on the item's path divides.
    __shared__ int s_item[2];
    __shared__ int4 s_crd[2];
    auto claim = [&](int slot) {
        const int item = (int)atomicAdd(p.counter, 1u);
        s_item[slot] = item;
        if (item < nitems) {
            const int bh = item / p.nchunks;
            s_crd[slot] = make_int4(bh / H, bh % H, p.chunk0 + item % p.nchunks, bh);
        }
    };
    // K and Q of the item in slot `slot`, with the expect_tx of every byte its
    // bars[0] phase counts (the g tile and the write key follow in issue_rest)
    auto issue_kq = [&](int slot) {
        const int4 c = s_crd[slot];
        const int b = c.x, h = c.y, n = c.z;
        mbar_arrive_expect_tx(&bars[0], (PD ? 6 : 4) * 8192 + (WK ? 2 * 8192 : 0));
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_3d_hint(sm + P_KQ + blk * 16384, &maps.k, &bars[0], h * D + 64 * blk, n * C, b, pol_in);
            tma_load_3d_hint(sm + P_KQ + blk * 16384 + 8192, &maps.q, &bars[0], h * D + 64 * blk, n * C, b, pol_in);
        }
    };
    // the rest of an item's tiles, into slots that are free only once the
    // previous item has finished: g (per-dimension gate; its slot held the
    // previous item's Qp staging), the write key, V
    auto issue_rest = [&](int b, int h, int n) {
        for (int blk = 0; blk < 2; ++blk) {
            if constexpr (PD)
                tma_load_3d_hint(sm + PD_KT + blk * 8192, &maps.g, &bars[0], h * D + 64 * blk, n * C, b, pol_in);
            if constexpr (WK)
                tma_load_3d_hint(sm + P_V + blk * 8192, &maps.kw, &bars[0], h * D + 64 * blk, n * C, b, pol_in);
        }
        if constexpr (!WK) {
            mbar_arrive_expect_tx(&bars[4], 2 * 8192);
            for (int blk = 0; blk < 2; ++blk)
                tma_load_3d_hint(sm + P_V + blk * 8192, &maps.v, &bars[4], h * D + 64 * blk, n * C, b, pol_in);
        }
    };
    // beta and g of an item, by warps 2-3 into registers
    float nb = 0.f, ng = 0.f;
    auto fetch_bg = [&](int slot) {
        const int4 c = s_crd[slot];
        const int b = c.x, h = c.y, n = c.z;
        const int t = n * C + (tid - 64);
        nb = ng = 0.f;
        if (t < T) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            nb = __bfloat162float(static_cast<const __nv_bfloat16*>(p.beta)[tok]);
            if constexpr (GATE == kGateScalar) ng = __bfloat162float(static_cast<const __nv_bfloat16*>(p.g)[tok]);
        }
    };

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        claim(0);
        if (s_item[0] < nitems) {
            issue_kq(0);
            if (EARLY) issue_rest(s_crd[0].x, s_crd[0].y, s_crd[0].z);
        }
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    int item = s_item[0];
    if ((warp == 2 || warp == 3) && item < nitems) fetch_bg(0);
    // the write key's tile: blocks of [64 tokens][64 d] with a stride of 8 KB
    // (WK, in the V slot) or the K tile's 16 KB (K and Q interleaved)
    const uint32_t kwo = WK ? P_V : P_KQ;
    const uint32_t kws = WK ? 8192u : 16384u;

#pragma unroll 1
    for (int it = 0; item < nitems; ++it) {
    ph = it & 1;
    const int4 crd = s_crd[it & 1];
    const int b = crd.x, h = crd.y, n = crd.z, bh = crd.w, nl = n - p.chunk0;
    uint8_t* img = p.ws + ((size_t)bh * p.cw + nl) * IMG_BYTES;
    // V into the slot the write key held, once every reader of the key is done
    // (the caller has passed a CTA barrier after the last read)
    auto load_v_late = [&]() {
        if constexpr (WK) {
            if (tid == 0) {
                fence_async_smem();
                mbar_arrive_expect_tx(&bars[4], 2 * 8192);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_3d_hint(sm + P_V + blk * 8192, &maps.v, &bars[4], h * D + 64 * blk, n * C, b, pol_in);
            }
        }
    };
    if (warp == 2 || warp == 3) {   // beta and g (fetched during the previous item)
        gbuf[tid - 64] = ng;
        sBeta[tid - 64] = nb;
    }
    __syncthreads();
    // the rest of the item's tiles, by a thread that is idle until the S
    // product is done (their slots were read by the previous item's stores
    // before the barrier at its end)
    if (!EARLY && tid == 160) issue_rest(b, h, n);
    // the next item, taken now so that the global atomic is off the path; its
    // K and Q are issued once this item's last readers of both are done
    if (tid == 64) claim((it + 1) & 1);

    bool exact = false;
    if constexpr (!PD) {
        if (warp == 0) chunk_gates<GATE>(gbuf, lane);
        if (tid == 32) {   // S = [K; Q] Kw^T (Kw = K without a separate write key)
            if (mbar_wait(&bars[0], ph, &failed)) {
                const uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t a = sb + P_KQ + (k >> 2) * 16384 + (k & 3) * 32;
                    const uint32_t bb = sb + kwo + (k >> 2) * kws + (k & 3) * 32;
                    mma_bf16(tmem + TM_S, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 16, 1024), id, k > 0);
                }
                mma_commit(&bars[1]);
            } else {
                atomicOr(p.status, kStatusTimeout);
            }
        }
        // the previous item's second Phi half (over the A scratch) is read
        if (tid == 128) bulk_wait_read();
        __syncthreads();
    } else {
        wait(0, ph);
        // G = in-chunk cumsum of g per key dimension by a segmented scan in
        // registers: lane pair (segment of 4 rows) x column group of 8
        // dimensions, then across the 16 segments; c = G_C per dimension.  The
        // reference c keeps every factor e^(G - c) below e^80 while the chunk
        // decays by less than that in every dimension; otherwise (exact) A and P
        // are formed on CUDA cores.
        const int cg = 2 * warp + (lane & 1), seg = lane >> 1;
        const int gblk = cg >> 3, gj = cg & 7, r0 = 4 * seg;
        float Gp[4][8], cv[8];
        bool wide = false;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + i;
            const uint4 raw = *reinterpret_cast<const uint4*>(sm + PD_KT + gblk * 8192 + r * 128 + ((gj ^ (r & 7)) * 16));
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(g2[e]);
                Gp[i][2 * e] = i ? Gp[i - 1][2 * e] + f.x : f.x;
                Gp[i][2 * e + 1] = i ? Gp[i - 1][2 * e + 1] + f.y : f.y;
            }
        }
        {
            float tot[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) tot[e] = Gp[3][e];
#pragma unroll
            for (int off = 2; off < 32; off <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float y = __shfl_up_sync(0xffffffffu, tot[e], off);
                    if (lane >= off) tot[e] += y;
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float ex = __shfl_up_sync(0xffffffffu, tot[e], 2);   // segments before this one
                if (lane < 2) ex = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) Gp[i][e] += ex;
                cv[e] = __shfl_sync(0xffffffffu, tot[e], 30 + (lane & 1));
                const float g0 = __shfl_sync(0xffffffffu, Gp[0][e], lane & 1);
                wide |= g0 - cv[e] >= 80.f;
            }
        }
        // the previous item's second Phi half (over the A / G scratch) is read
        if (tid == 128) bulk_wait_read();
        exact = __syncthreads_or(wide) != 0;
        if (seg == 15) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gm = expf(cv[e]);
                sGamD[8 * cg + e] = gm;
                sRef[8 * cg + e] = exact ? 1.f : gm;
            }
        }
        // K~ = K e^(c - G), written transposed (K~^T [d][i]) over the g tile, which
        // every thread has read before the barrier above; factored: K e^(G - c),
        // Q e^(G - c) in place; exact: G kept
        float ktv[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = r0 + i;
            const uint32_t ro = r * 128 + ((gj ^ (r & 7)) * 16);
            uint8_t* kp = sm + P_KQ + gblk * 16384 + ro;
            const uint4 kraw = *reinterpret_cast<const uint4*>(kp);
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kraw);
            const uint4 wraw = *reinterpret_cast<const uint4*>(sm + kwo + gblk * kws + ro);
            const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&wraw);
            if (!exact) {
                const uint4 qraw = *reinterpret_cast<const uint4*>(kp + 8192);
                const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qraw);
                uint32_t kc[4], qc[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __bfloat1622float2(k2[e]);
                    const float2 qf = __bfloat1622float2(q2[e]);
                    const float x0 = Gp[i][2 * e] - cv[2 * e], x1 = Gp[i][2 * e + 1] - cv[2 * e + 1];
                    const float f0 = __expf(x0), f1 = __expf(x1);
                    const float b0 = __expf(-x0), b1 = __expf(-x1);
                    const float2 wf = __bfloat1622float2(w2[e]);
                    kc[e] = pack_bf16(kf.x * f0, kf.y * f1);
                    qc[e] = pack_bf16(qf.x * f0, qf.y * f1);
                    ktv[i][2 * e] = wf.x * b0;
                    ktv[i][2 * e + 1] = wf.y * b1;
                }
                *reinterpret_cast<uint4*>(kp) = make_uint4(kc[0], kc[1], kc[2], kc[3]);
                *reinterpret_cast<uint4*>(kp + 8192) = make_uint4(qc[0], qc[1], qc[2], qc[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 wf = __bfloat1622float2(w2[e]);
                    ktv[i][2 * e] = wf.x * __expf(cv[2 * e] - Gp[i][2 * e]);
                    ktv[i][2 * e + 1] = wf.y * __expf(cv[2 * e + 1] - Gp[i][2 * e + 1]);
                }
                float* grow = Gs + r * LDG + 8 * cg;
                *reinterpret_cast<float4*>(grow) = make_float4(Gp[i][0], Gp[i][1], Gp[i][2], Gp[i][3]);
                *reinterpret_cast<float4*>(grow + 4) = make_float4(Gp[i][4], Gp[i][5], Gp[i][6], Gp[i][7]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)   // row d of K~^T, columns i = r0 .. r0 + 3
            *reinterpret_cast<uint2*>(sm + PD_KT + sw128_offset(8 * cg + e, r0)) =
                make_uint2(pack_bf16(ktv[0][e], ktv[1][e]), pack_bf16(ktv[2][e], ktv[3][e]));
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 64 && !failed) {   // K~^T is final: its image goes out now
            bulk_store_hint(img + IMG_KP, sm + PD_KT, 16384, pol_img);
            bulk_commit();
        }
        if (!exact && tid == 32) {   // S = [K e^(G-c); Q e^(G-c)] K~^T (B MN-major: K~^T [d][i])
            const uint32_t id = idesc_bf16_f32(128, 64, false, true);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = sb + P_KQ + (k >> 2) * 16384 + (k & 3) * 32;
                const uint32_t bb = sb + PD_KT + k * 2048;
                mma_bf16(tmem + TM_S, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), id, k > 0);
            }
            mma_commit(&bars[1]);
        } else if (exact && tid == 32) {
            mbar_arrive(&bars[1]);   // no product: complete the phase, so that every
                                     // barrier completes once per item
        }
    }

    // ---- A (fp32 scratch) and P (bf16, K-major [r][i]) from S
    {
        const int q4 = warp & 3, ch = warp >> 2;
        const int L = q4 * 32 + lane;
        float sv[32];
        if (!exact) {
            wait(1, ph);
            tc_fence_after();
            ld_cols<32>(tmem + TM_S + lane_off + 32 * ch, sv);
            const float* sG = gbuf;
            const float* sU = gbuf + 256;
            const float* sW = gbuf + 320;
            const bool fact = PD || gbuf[384] != 0.f;
            // row r of A (lanes 0-63, strictly lower) or of P (lanes 64-127,
            // inclusive); the per-column factors w_i (or G_i) are read four at a
            // time (the same address across the warp: one broadcast load)
            const bool isp = L >= 64;
            const int r = isp ? L - 64 : L;
            const int lim = isp ? r + 1 : r;      // columns i < lim are kept
            const float* colf = (fact ? sW : sG) + 32 * ch;
            if (fact) {
                const float cr = isp ? (PD ? 1.f : sU[r]) : (PD ? sBeta[r] : sBeta[r] * sU[r]);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 w4 = PD ? make_float4(1.f, 1.f, 1.f, 1.f)
                                         : *reinterpret_cast<const float4*>(colf + 4 * j);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int e = 4 * j + t;
                        sv[e] = (32 * ch + e < lim) ? cr * wv[t] * sv[e] : 0.f;
                    }
                }
            } else {
                const float Gr = sG[r], br = isp ? 1.f : sBeta[r];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 g4 = *reinterpret_cast<const float4*>(colf + 4 * j);
                    const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int e = 4 * j + t;
                        sv[e] = (32 * ch + e < lim) ? br * __expf(Gr - gv[t]) * sv[e] : 0.f;
                    }
                }
            }
        } else if constexpr (PD) {
            // exact A and P: sum_d k_rd k_id e^(G_rd - G_id) with every exponent <= 0
            const int r = L & 63;
            const bool isq = L >= 64;
            const uint8_t* rowt = sm + P_KQ + (isq ? 8192 : 0);
#pragma unroll 1
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * ch + e;
                float acc = 0.f;
                if (isq ? (i <= r) : (i < r)) {
#pragma unroll 4
                    for (int d = 0; d < D; ++d) {
                        const float x = ld_bf16(rowt + (d >> 6) * 16384, r, d & 63);
                        const float kk = ld_bf16(sm + kwo + (d >> 6) * kws, i, d & 63);
                        acc = fmaf(x * kk, expf(Gs[r * LDG + d] - Gs[i * LDG + d]), acc);
                    }
                }
                sv[e] = isq ? acc : sBeta[r] * acc;
            }
            __syncthreads();   // raw K, Q and G read by every thread
            {   // reference 0: K e^G, Q e^G in place (same elements as the scan's)
                const int cg = 2 * warp + (lane & 1), r0 = 4 * (lane >> 1);
                const int gblk = cg >> 3, gj = cg & 7;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = r0 + i;
                    uint8_t* kp = sm + P_KQ + gblk * 16384 + r * 128 + ((gj ^ (r & 7)) * 16);
                    const uint4 kraw = *reinterpret_cast<const uint4*>(kp);
                    const uint4 qraw = *reinterpret_cast<const uint4*>(kp + 8192);
                    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kraw);
                    const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qraw);
                    const float* grow = Gs + r * LDG + 8 * cg;
                    uint32_t kc[4], qc[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 kf = __bfloat1622float2(k2[e]);
                        const float2 qf = __bfloat1622float2(q2[e]);
                        const float f0 = __expf(grow[2 * e]), f1 = __expf(grow[2 * e + 1]);
                        kc[e] = pack_bf16(kf.x * f0, kf.y * f1);
                        qc[e] = pack_bf16(qf.x * f0, qf.y * f1);
                    }
                    *reinterpret_cast<uint4*>(kp) = make_uint4(kc[0], kc[1], kc[2], kc[3]);
                    *reinterpret_cast<uint4*>(kp + 8192) = make_uint4(qc[0], qc[1], qc[2], qc[3]);
                }
            }
            __syncthreads();   // G (aliased with A) is dead from here on
        }
        if (L < 64) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(Af + L * LDF + 32 * ch + e) =
                    make_float4(sv[e], sv[e + 1], sv[e + 2], sv[e + 3]);
        } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) st_row_chunk(sm + P_P, L - 64, 4 * ch + jj, sv + 8 * jj, 1.f);
        }
    }
    __syncthreads();
    if constexpr (PD) load_v_late();   // the write key's last reader was the scan / exact A, P
    forward_substitution(Af, Tf, tid, [&](int t) {
        if constexpr (!PD) {   // K~^T [d][i] = (diag(e^(G_C - G_i)) K)^T into its own tile
            const float* sFt = gbuf + 128;
#pragma unroll 1
            for (int idx = t; idx < 512; idx += NPR - 64) {   // (token pair, 8 dims) items
                const int ip = idx & 31, dc = idx >> 5;
                const int i0 = 2 * ip, blk = dc >> 3, j = dc & 7;
                const uint8_t* kb = sm + kwo + blk * kws;
                uint4 r0 = *reinterpret_cast<const uint4*>(kb + i0 * 128 + ((j ^ (i0 & 7)) * 16));
                uint4 r1 = *reinterpret_cast<const uint4*>(kb + (i0 + 1) * 128 + ((j ^ ((i0 + 1) & 7)) * 16));
                const float f0 = sFt[i0], f1 = sFt[i0 + 1];
                const __nv_bfloat16* e0 = reinterpret_cast<const __nv_bfloat16*>(&r0);
                const __nv_bfloat16* e1 = reinterpret_cast<const __nv_bfloat16*>(&r1);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<uint32_t*>(sm + P_KT + sw128_offset(8 * dc + e, i0)) =
                        pack_bf16(__bfloat162float(e0[e]) * f0, __bfloat162float(e1[e]) * f1);
            }
            fence_async_smem();
            named_bar(5, NPR - 64);
            if (t == 0 && !failed) {   // K~^T is final: its image goes out now (thread 64)
                bulk_store_hint(img + IMG_KP, sm + P_KT, 16384, pol_img);
                bulk_commit();
            }
        }
    });
    if constexpr (!PD) load_v_late();  // K~^T, the write key's last reader, is formed
    // T diag(beta) and T diag(beta e^G) as bf16 K-major [r][i]
    {
        const float* sGam = gbuf + 64;
        const int r = tid >> 2, j0 = 2 * (tid & 3);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = j0 + jj;
            const float4 t0 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j);
            const float4 t1 = *reinterpret_cast<const float4*>(Tf + r * LDF + 8 * j + 4);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            const float4 b0 = *reinterpret_cast<const float4*>(sBeta + 8 * j);
            const float4 b1 = *reinterpret_cast<const float4*>(sBeta + 8 * j + 4);
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float gv[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
            if constexpr (!PD) {
                const float4 g0 = *reinterpret_cast<const float4*>(sGam + 8 * j);
                const float4 g1 = *reinterpret_cast<const float4*>(sGam + 8 * j + 4);
                gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w;
                gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
            }
            float tu[8], tw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * j + e;
                tu[e] = (i <= r) ? tv[e] * bv[e] : 0.f;
                tw[e] = tu[e] * gv[e];
            }
            st_row_chunk(sm + P_TU, r, j, tu, 1.f);
            if constexpr (!PD) st_row_chunk(sm + P_TW, r, j, tw, 1.f);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 32 && !failed) {
        // W^T = (K e^G)^T T_w^T, U^T = V^T T_u^T.  Scalar gate: the decay sits in
        // T_w; per-dimension gate: (K e^(G-ref))^T T_u^T, rows d times e^(ref_d)
        // in the epilogue
        const uint32_t id = idesc_bf16_f32(128, 64, true, false);
        const uint32_t tw = PD ? sb + P_TU : sb + P_TW;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mma_bf16(tmem + TM_WT, sdesc_sw128(sb + P_KQ + k * 2048, 16384, 1024),
                     sdesc_sw128(tw + k * 32, 16, 1024), id, k > 0);
        if (!mbar_wait(&bars[4], ph, &failed)) atomicOr(p.status, kStatusTimeout);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mma_bf16(tmem + TM_UT, sdesc_sw128(sb + P_V + k * 2048, 8192, 1024),
                     sdesc_sw128(sb + P_TU + k * 32, 16, 1024), id, k > 0);
        mma_commit(&bars[2]);
    }
    wait(2, ph);
    tc_fence_after();
    {   // [W^T; U^T] as one K-major bf16 tile of 256 rows (tokens contiguous)
        const int row = (warp & 3) * 32 + lane;
        const float sc = (PD && warp < 4) ? sRef[row] : 1.f;
        float v[64];
        ld_cols<64>(tmem + (warp < 4 ? TM_WT : TM_UT) + lane_off, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) st_row_chunk(sm + P_WUT, (warp < 4 ? 0 : 128) + row, j, v + 8 * j, sc);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && !failed) {   // U^T and P are final
        bulk_store_hint(img + IMG_UT, sm + P_WUT + 16384, 16384, pol_img);
        bulk_store_hint(img + IMG_KP + 16384, sm + P_P, 8192, pol_img);
        bulk_commit();
    }
    if (tid == 32 && !failed) {
        const uint32_t kt = sb + P_KT;
        const uint32_t id1 = idesc_bf16_f32(128, 128, false, false);   // K~^T W (both K-major)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mma_bf16(tmem + TM_FP, sdesc_sw128(kt + k * 32, 16, 1024),
                     sdesc_sw128(sb + P_WUT + k * 32, 16, 1024), id1, k > 0);
        // P W (B = W^T as for K~^T W): the A operand starts at row 64 of K~^T, so
        // that its rows 64..127 are P (the tile after K~^T); lanes 0..63 of the
        // result are not used
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mma_bf16(tmem + TM_PW, sdesc_sw128(kt + 8192 + k * 32, 16, 1024),
                     sdesc_sw128(sb + P_WUT + k * 32, 16, 1024), id1, k > 0);
        mma_commit(&bars[3]);
    }
    wait(3, ph);
    // Row r of Q (its half hh of the columns) into the registers of the thread
    // that forms row r of Qp (lanes 64 + r), so that the next item's K and Q
    // can land once every thread has passed the barrier below.  The K~^T tile
    // becomes the Qp staging: its image store (issued by thread 64) must have
    // read it.
    const int row = (warp & 3) * 32 + lane;
    uint4 qrow[8];
    if (row >= 64) {
        const uint8_t* qb = sm + P_KQ + 8192 + (warp >> 2) * 16384;
#pragma unroll
        for (int j = 0; j < 8; ++j) qrow[j] = *reinterpret_cast<const uint4*>(qb + sw128_offset(row - 64, 8 * j));
    }
    if (tid == 64) bulk_wait_read();   // K~^T's image store (thread 64's only group)
    tc_fence_after();
    __syncthreads();
    const int next_item = s_item[(it + 1) & 1];
    if ((warp == 2 || warp == 3) && next_item < nitems) fetch_bg((it + 1) & 1);
    {   // Phi = -K~^T W, row d: warps 0-3 columns 0-63, warps 4-7 columns 64-127;
        // each half stored as soon as it is staged
        const int hh = warp >> 2;
        float v[64];
        ld_cols<64>(tmem + TM_FP + lane_off + 64 * hh, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) st_row_chunk(sm + S_PHI + hh * 16384, row, j, v + 8 * j, -1.f);
        fence_async_smem();
        if (hh == 0) named_bar(1, 128);
        else named_bar(3, 128);
        if ((tid & 127) == 0 && !failed) {
            bulk_store_hint(img + IMG_PQ + hh * PQ_BLK, sm + S_PHI + hh * 16384, 16384, pol_img);
            bulk_commit();
        }
        // the next item's K and Q: every reader of this item's is done (the Q
        // rows of Qp were read before the barrier above); issued by a thread
        // whose warps have no Qp rows, after its share of Phi
        if (tid == 0 && next_item < nitems) {
            fence_async_smem();
            issue_kq((it + 1) & 1);
        }
    }
    if (warp >= 4 && !failed) {   // gamma_d, d = row
        float gam;
        if constexpr (PD) gam = sGamD[row];
        else gam = gbuf[64 + 63];   // e^(G_C); 1 without a gate
        reinterpret_cast<float*>(img + IMG_GAM)[row] = gam;
    }
    if (row >= 64) {   // Qp = Q e^G - P W, row r, columns 64 hh ..: K-major [r][d] (two
                       // [64][64] blocks), 16-byte chunks
        const int hh = warp >> 2, r = row - 64;
        float v[64];
        ld_cols<64>(tmem + TM_PW + lane_off + 64 * hh, v);
        const float er = gbuf[64 + r];   // e^(G_r); 1 without a gate
        uint8_t* qblk = sm + S_QPT + hh * 8192;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const __nv_bfloat16* q8 = reinterpret_cast<const __nv_bfloat16*>(&qrow[j]);
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float qs = PD ? sRef[64 * hh + 8 * j + e] : er;
                x[e] = fmaf(qs, __bfloat162float(q8[e]), -v[8 * j + e]);
            }
            st_row_chunk(qblk, r, j, x, 1.f);
        }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        if (!failed) {
            bulk_store_hint(img + IMG_PQ + 16384, sm + S_QPT, 8192, pol_img);
            bulk_store_hint(img + IMG_PQ + PQ_BLK + 16384, sm + S_QPT + 8192, 8192, pol_img);
            bulk_commit();
        }
        // every staging of this item is read (Phi's first half is over the V
        // slot, Qp's over the g slot and K~^T: the next item loads V and g first)
        bulk_wait_read();
        rest_issued = false;
        if (EARLY && next_item < nitems && !failed) {
            const int4 c = s_crd[(it + 1) & 1];
            fence_async_smem();
            issue_rest(c.x, c.y, c.z);
            rest_issued = true;
        }
    }
    tc_fence_before();
    if (__syncthreads_or(failed)) {
        // a bounded wait gave up: wait (bounded) for this item's loads and the
        // next item's K and Q, if they were issued, then take no more items
        if (tid == 0) {
            int f2 = 0;
            const bool cur = mbar_wait(&bars[0], ph, &f2);
            mbar_wait(&bars[4], ph, &f2);
            if (cur && next_item < nitems) mbar_wait(&bars[0], ph ^ 1u, &f2);
            if (rest_issued && !WK) mbar_wait(&bars[4], ph ^ 1u, &f2);
        }
        __syncthreads();
        break;
    }
    tc_fence_after();
    item = next_item;
    }   // items
    if (tid == 0 || tid == 64 || tid == 128) bulk_wait_all();   // the last item's stores are complete
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ chain
// The chain runs on the transposed state: h^T [v][d] (fp32 in the state-pass
// registers, its bf16 copy in TMEM as the A operand of the state product), so
// that neither the state's bf16 copy nor the product's h operand touch shared
// memory.  Per chunk n, into one accumulator D_n of 192 columns (M = 128 v):
//   D_n  = U_n^T [K~_n | P_n^T]        (N = 192, K = 64 tokens; A = U^T from shared memory)
//   D_n += h_n^T [Phi_n^T | Qp_n^T]    (N = 192, K = 128; A = h^T from TMEM)
// Columns 0..127 of D_n are X^T_n = U^T K~ + h^T Phi^T, so the state pass forms
//   h_{n+1}^T = h_n^T Diag(gamma_n) + X^T_n
// and columns 128..191 are O^T_n = U^T P^T + h^T Qp^T, the chunk's output.
// Only the second product is on the serial path; U^T [K~ | P^T] needs no
// state and is issued a chunk ahead by its own warp, so that it runs while the
// state pass works.  The tensor pipe takes ~80-140 cycles per instruction
// whatever N up to 256 and a satisfied mbarrier wait costs ~100-200 cycles, so
// the serial loop has one product of 8 instructions, one wait on the state
// product's completion, and one named barrier from the state pass to the
// issuing thread.

// Chain kernel shared memory (bytes from a 1 KB-aligned base).
constexpr uint32_t CH_PQ = 0;           // 2 slots of [Phi ; Qp] (48 KB each); the final state's staging
constexpr uint32_t CH_KP = 98304;       // 2 slots of [K~^T ; P] (24 KB each)
constexpr uint32_t CH_UT = 147456;      // 2 slots of U^T (16 KB each)
constexpr uint32_t CH_OT = 180224;      // 2 slots of the O tile [r][64 v] x 2 blocks for its TMA store
constexpr uint32_t CH_GAM = 212992;     // 4 slots of gamma (512 B each)
constexpr uint32_t CH_BAR = 215040;
constexpr uint32_t CH_SMEM = CH_BAR + 512 + 1024;
static_assert(CH_SMEM <= 232448, "chain shared memory");
static_assert(CH_KP == 2 * 2 * PQ_BLK && CH_UT == CH_KP + 2 * 24576 && CH_OT == CH_UT + 2 * 16384,
              "chain slots");

constexpr int CH_THREADS = 736;   // 23 warps: loader, 2 MMA issuers, 4 output, 16 state
constexpr int W_UK = 2;           // issuer of U^T [K~ | P^T]
constexpr int W_OUT = 3;          // first output warp
constexpr int W_ST = 7;           // first state-pass warp
constexpr int N_ST = 16;          // state-pass warps: lane quarter (v) x column quarter (d)
constexpr int BAR_H = 3;          // named barrier: h^T of the chunk is in TMEM (state pass ->
                                  //   state-product issuer)
// Registers: warps spread over the SM's four sub-partitions of 16 K registers
// each, so 23 warps (six on three sub-partitions) allow at most 85 a thread,
// 80 in the allocation granularity of 8.

// TMEM columns of the chain kernel (512 allocated): slot s of D at 256 s
// (192 columns: X^T then O^T), slot s of the bf16 h^T at 192 + 256 s (lanes v,
// d pairs packed two to a 32-bit column).
constexpr uint32_t TM_D = 0;
constexpr uint32_t TM_HT = 192;
constexpr uint32_t TM_SLOT = 256;

enum ChainBar {
    CB_KU0, CB_KU1, CB_PQ0, CB_PQ1, CB_GAM0, CB_GAM1, CB_GAM2, CB_GAM3, CB_KUFREE0, CB_KUFREE1,
    CB_PQFREE0, CB_PQFREE1, CB_SDONE0, CB_SDONE1, CB_ODONE0, CB_ODONE1,
    CB_XFREE0, CB_XFREE1, CB_OFREE0, CB_OFREE1, CB_FINAL, CB_COUNT
};
static_assert(CB_COUNT * 8 <= 512, "barrier space");

// Tensor maps of the chain kernel: o (bf16, [B][T][H*D], 64 x 64 boxes) and the
// final state (fp32, [B*H][D][D], boxes of 128 rows x 32 columns = 128 B,
// swizzled so that the lanes of a warp -- 32 consecutive columns v of one
// row d -- write one row of a box without bank conflicts).
struct ChainMaps {
    CUtensorMap o, s_out;
    CUtensorMap seg;   // [2][B*H][nseg][D][D] segment offsets then transitions (segment mode 1)
};


// Element (d, v) of the final state staged as four TMA boxes of [128 d][32 v]
// fp32 (128-byte swizzle), box v / 32.
__device__ __forceinline__ uint32_t st_off(int d, int v) {
    return (uint32_t)(v >> 5) * 16384u + (uint32_t)d * 128u +
           ((uint32_t)(((v & 31) >> 2) ^ (d & 7)) << 4) + ((uint32_t)(v & 3) << 2);
}

// One CTA per (batch, head): walks the wave's chunks in order.  Roles:
//   warp 0       loader: [K~^T ; P] and U^T, then [Phi ; Qp] and gamma, two
//                chunks ahead, by bulk copies; L2 prefetch and discard
//   warp 1       state-product issuer: h^T [Phi^T | Qp^T] of chunk n as soon as
//                the state pass has written h^T (named barrier BAR_H)
//   warp 2       U^T [K~ | P^T] of chunk n + 1 as soon as its slot of D is free,
//                so it runs while the state pass of chunk n works
//   warps 3-6    output: O^T from TMEM -> the bf16 O tile -> TMA store
//   warps 7-22   state pass (lane quarter x column quarter of d)
// Every mbarrier is per slot (or per gamma slot) and completes at most once
// ahead of its wait, so no parity wait can fall two phases behind; the state
// pass and the state-product issuer alternate on BAR_H (the pass of chunk
// n + 1 needs the product of chunk n).
// UNIFORM_GAMMA: every column of the state decays by the same gamma (scalar gate
// or none), so the state pass reads one value per chunk, ahead of the product.
template <bool UNIFORM_GAMMA>
__global__ void __maxnreg__(80)
chunk_chain_kernel(const __grid_constant__ ChainMaps maps, const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + CH_BAR);
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    // Role of this CTA.  Plain mode: one CTA per (batch, head) over the wave,
    // from the entering state, with outputs.  Segment mode 1: per (batch, head,
    // segment) the segment's offset (from a zero state, role 1) and, in the
    // second half of the grid, its transition (from the identity with no
    // writes, role 2), no outputs.  Segment mode 3: per (batch, head, segment)
    // the outputs from the segment's entering state (role 0).
    const int nbh = p.B * p.H;
    const int S = p.seg_mode ? p.nseg : 1;
    int role = 0, bh = blockIdx.x, j = 0;
    if (p.seg_mode == 1) {
        const int per = nbh * S;
        role = (int)blockIdx.x < per ? 1 : 2;
        const int r = (int)blockIdx.x % per;
        bh = r / S;
        j = r % S;
    } else if (p.seg_mode == 3) {
        bh = blockIdx.x / S;
        j = blockIdx.x % S;
    }
    const int b = bh / H, h = bh % H;
    const int c0 = p.seg_mode ? j * p.seg_len : 0;
    const int NC = p.seg_mode ? min(p.seg_len, p.nchunks - c0) : p.nchunks;
    const bool outputs = role == 0;
    const uint8_t* wsh = p.ws + ((size_t)bh * p.cw + c0) * IMG_BYTES;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint64_t pol_once = l2_evict_first();   // images (dead once read) and o
    int failed = 0;

    if (tid == 0) {
        for (int i = 0; i < CB_COUNT; ++i)
            mbar_init(&bars[i], (i == CB_XFREE0 || i == CB_XFREE1) ? N_ST : 1);
        fence_mbar_init();
        prefetch_tmap(&maps.o);
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    // the next wave's prep may start on the SMs this grid leaves idle; the
    // images and the carried state of this wave are read only after the wait.
    // (The segment offsets and transitions let the combine start only once
    // they are done: its CTAs must not hold SMs that theirs still need.)
    if (p.seg_mode != 1) pdl_launch_dependents();
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    auto wait = [&](int bar, uint32_t parity) {
        if (!mbar_wait(&bars[bar], parity, &failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    };
    auto img = [&](int nl) { return wsh + (size_t)nl * IMG_BYTES; };

    if (warp == 0) {
        // =========================== loader: [K~^T ; P] and U^T, [Phi ; Qp] (2 slots
        // each, two chunks ahead), gamma (4 slots); each image prefetched into L2
        // two chunks ahead, its lines dropped from L2 once loaded and used
        if (lane == 0) {
            for (int nl = 0; nl < 2 && nl < NC; ++nl) bulk_prefetch_l2(img(nl), IMG_BYTES);
        }
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            if (role != 2) {   // the transition (role 2) writes nothing: no K~^T, P, U^T
            if (nl >= 2) wait(CB_KUFREE0 + s, ((nl - 2) >> 1) & 1);   // U^T [K~|P^T] of nl - 2 done
            if (failed) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[CB_KU0 + s], 24576 + 16384);
                bulk_load_hint(sm + CH_KP + s * 24576, img(nl) + IMG_KP, 24576, &bars[CB_KU0 + s], pol_once);
                bulk_load_hint(sm + CH_UT + s * 16384, img(nl) + IMG_UT, 16384, &bars[CB_KU0 + s], pol_once);
            }
            }
            if (nl >= 2) wait(CB_PQFREE0 + s, ((nl - 2) >> 1) & 1);   // state product of nl - 2 done
            if (failed) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[CB_PQ0 + s], 2 * PQ_BLK);
                bulk_load_hint(sm + CH_PQ + s * 2 * PQ_BLK, img(nl) + IMG_PQ, 2 * PQ_BLK, &bars[CB_PQ0 + s], pol_once);
                mbar_arrive_expect_tx(&bars[CB_GAM0 + (nl & 3)], 512);
                bulk_load_hint(sm + CH_GAM + (nl & 3) * 512, img(nl) + IMG_GAM, 512, &bars[CB_GAM0 + (nl & 3)], pol_once);
                if (nl + 2 < NC) bulk_prefetch_l2(img(nl + 2), IMG_BYTES);
            }
            if (nl >= 2 && outputs && !p.h_all) {   // both products of chunk nl - 2 are done:
                             // its image is dead in L2 (gamma of chunk nl - 3 too: the state
                             // pass has used it); segment offsets and transitions leave them for
                             // the outputs, and the backward's forward keeps them all
                l2_discard(img(nl - 2), IMG_GAM, lane);
                if (nl >= 3) l2_discard(img(nl - 3) + IMG_GAM, 512, lane);
            }
        }
    } else if (warp == 1) {
        // =========================== state-product issuer: D_nl += h^T [Phi^T | Qp^T]
        // (N = 128 without outputs) once the state pass has written h^T; the
        // waits that are normally satisfied by then come before the barrier
        const bool leader = lane == 0;
        const uint32_t id = idesc_bf16_f32(128, outputs ? 192 : 128, false, false);
        const uint64_t d_pq = sdesc_sw128(sb + CH_PQ, 16, 1024);
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            wait(CB_PQ0 + s, (nl >> 1) & 1);
            if (role != 2) wait(CB_KUFREE0 + s, (nl >> 1) & 1);   // U^T [K~ | P^T] of nl is in D
            named_bar(BAR_H, 32 + 32 * N_ST);                        // h^T of nl is in TMEM
            tc_fence_after();
            if (leader && !failed) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ta(tmem + TM_D + TM_SLOT * s, tmem + TM_HT + TM_SLOT * s + 8 * k,
                                d_pq + ((s * 2 * PQ_BLK + (k >> 2) * PQ_BLK + (k & 3) * 32) >> 4),
                                id, role != 2 || k > 0);   // the transition has no U^T K~
                mma_commit(&bars[CB_SDONE0 + s]);
                if (outputs) mma_commit(&bars[CB_ODONE0 + s]);
                mma_commit(&bars[CB_PQFREE0 + s]);
            }
        }
        if (leader) mma_commit(&bars[CB_FINAL]);
        int final_failed = 0;
        if (!mbar_wait(&bars[CB_FINAL], 0, &final_failed)) atomicOr(p.status, kStatusTimeout);
        __syncwarp();
    } else if (warp == W_UK) {
        // =========================== D_nl = U^T [K~ | P^T] once its operands are in
        // and both readers of D in this slot (state pass and output, chunk
        // nl - 2) are done with it; runs a chunk ahead of the state product
        const bool leader = lane == 0;
        const uint32_t id = idesc_bf16_f32(128, 192, false, false);
        const uint64_t d_kp = sdesc_sw128(sb + CH_KP, 16, 1024);
        const uint64_t d_ut = sdesc_sw128(sb + CH_UT, 16, 1024);
#pragma unroll 1
        for (int nl = 0; nl < (role != 2 ? NC : 0); ++nl) {
            const int s = nl & 1;
            wait(CB_KU0 + s, (nl >> 1) & 1);
            if (nl >= 2) {
                wait(CB_XFREE0 + s, ((nl - 2) >> 1) & 1);
                if (outputs) wait(CB_OFREE0 + s, ((nl - 2) >> 1) & 1);
            }
            tc_fence_after();
            if (leader && !failed) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem + TM_D + TM_SLOT * s, d_ut + ((s * 16384 + k * 32) >> 4),
                             d_kp + ((s * 24576 + k * 32) >> 4), id, k > 0);
                mma_commit(&bars[CB_KUFREE0 + s]);
            }
            __syncwarp();
        }
    } else if (warp < W_ST) {   // warps W_OUT ..
        // =========================== output: O^T row v -> the O tile [r][v]
        // (bf16, swizzled) in its slot -> TMA store
        const int v = (warp & 3) * 32 + lane;
        const bool leader = warp == W_OUT && lane == 0;
#pragma unroll 1
        for (int nl = 0; nl < (outputs ? NC : 0); ++nl) {
            const int s = nl & 1;
            if (leader && nl >= 2) bulk_wait_read_all_but_one();   // the store of chunk nl - 2 read slot s
            named_bar(2, 128);
            wait(CB_ODONE0 + s, (nl >> 1) & 1);
            tc_fence_after();
            uint8_t* ot = sm + CH_OT + s * 16384 + (v >> 6) * 8192;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float ov[32];
                ld_cols<32>(tmem + TM_D + TM_SLOT * s + 128 + 32 * half + lane_off, ov);
#pragma unroll
                for (int r = 0; r < 32; ++r)
                    *reinterpret_cast<__nv_bfloat16*>(ot + sw128_offset(32 * half + r, v & 63)) =
                        __float2bfloat16_rn(ov[r]);
            }
            fence_async_smem();
            tc_fence_before();
            named_bar(2, 128);
            if (leader) {
                mbar_arrive(&bars[CB_OFREE0 + s]);
                if (!failed) {
                    const int t0 = (p.chunk0 + c0 + nl) * C;
                    tma_store_3d_hint(&maps.o, sm + CH_OT + s * 16384, h * D, t0, b, pol_once);
                    tma_store_3d_hint(&maps.o, sm + CH_OT + s * 16384 + 8192, h * D + 64, t0, b, pol_once);
                    bulk_commit();
                }
            }
        }
        if (leader) bulk_wait_all();
    } else {
        // =========================== state pass: h'^T = h^T Diag(gamma) + X^T in
        // fp32 registers (row v, columns d = 32c..), its bf16 copy into TMEM
        const int v = (warp & 3) * 32 + lane;
        const int c = (warp - W_ST) >> 2;           // column quarter of d
        float hv[32];
        // hv = h_{nl-1}^T Diag(gamma_{nl-1}) + X^T_{nl-1}, once the state product of
        // chunk nl - 1 is done; a uniform gamma is read before that wait
        // (the decay is applied while the product is still running, so that only
        // the additions follow its completion)
        auto advance = [&](int nl) {
            const int sp = (nl - 1) & 1;
            const float* gp = reinterpret_cast<const float*>(sm + CH_GAM + ((nl - 1) & 3) * 512) + 32 * c;
            wait(CB_GAM0 + ((nl - 1) & 3), ((nl - 1) >> 2) & 1);
            if constexpr (UNIFORM_GAMMA) {
                const float g1 = *gp;
#pragma unroll
                for (int e = 0; e < 32; ++e) hv[e] *= g1;
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 g4 = *reinterpret_cast<const float4*>(gp + 4 * j);
                    hv[4 * j] *= g4.x;
                    hv[4 * j + 1] *= g4.y;
                    hv[4 * j + 2] *= g4.z;
                    hv[4 * j + 3] *= g4.w;
                }
            }
            wait(CB_SDONE0 + sp, ((nl - 1) >> 1) & 1);
            tc_fence_after();
            float xv[32];
            ld_cols<32>(tmem + TM_D + TM_SLOT * sp + lane_off + 32 * c, xv);
#pragma unroll
            for (int e = 0; e < 32; ++e) hv[e] += xv[e];
        };
#pragma unroll 1
        for (int nl = 0; nl < NC; ++nl) {
            const int s = nl & 1;
            if (nl == 0) {
                // the entering state: the wave's (plain mode, first segment), the
                // segment's from the combine (later segments), zero (offsets) or
                // the identity (transitions)
                const float* s0 = role != 0 ? nullptr
                                  : j == 0  ? (p.s0 ? p.s0 + (size_t)bh * D * D : nullptr)
                                            : p.seg_h + ((size_t)bh * S + j) * D * D;
                if (s0) {   // column v, rows d = 32c.. of M = S^T: for each d the 32
                            // lanes read 128 consecutive bytes (L2 only: the carried
                            // state was written by an earlier launch)
                    const float* src = s0 + (size_t)(32 * c) * D + v;
#pragma unroll
                    for (int e = 0; e < 32; ++e) hv[e] = __ldcg(src + (size_t)e * D);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) hv[e] = (role == 2 && 32 * c + e == v) ? 1.f : 0.f;
                }
            } else {
                advance(nl);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[CB_XFREE0 + ((nl - 1) & 1)]);
            }
            if (p.h_all) {   // keep the chunk's entering state (fp32) for the backward
                float* dst = p.h_all + ((size_t)bh * p.nc_total + p.chunk0 + c0 + nl) * D * D +
                             (size_t)(32 * c) * D + v;
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[(size_t)e * D] = hv[e];
            }
            {
                float pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = __uint_as_float(pack_bf16(hv[2 * e], hv[2 * e + 1]));
                tmem_st16(tmem + TM_HT + TM_SLOT * s + 16 * c + lane_off, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            named_bar_arrive(BAR_H, 32 + 32 * N_ST);
        }
        if (NC > 0) {   // final state, staged over the [Phi ; Qp] slots (free once the
                        // last state product is done), written by four TMA stores
            advance(NC);
            // where the final state goes: the wave's (plain mode, last segment), the
            // segment's offset or transition (segment mode 1), or nowhere
            const CUtensorMap* smap = role != 0 ? &maps.seg : (j == S - 1 ? &maps.s_out : nullptr);
            const int sidx = role == 0 ? bh : (role - 1) * nbh * S + bh * S + j;
            if (role != 0 || (j == S - 1 && p.s_out)) {
                // the last chunk's h^T Qp^T (behind h^T Phi^T) may still read its slot
                if (outputs) wait(CB_ODONE0 + ((NC - 1) & 1), ((NC - 1) >> 1) & 1);
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    *reinterpret_cast<float*>(sm + CH_PQ + st_off(32 * c + e, v)) = hv[e];
                fence_async_smem();
                named_bar(1, 32 * N_ST);
                if (warp == W_ST && lane == 0) {
                    if (!failed) {
                        for (int cb = 0; cb < 4; ++cb)
                            tma_store_3d(smap, sm + CH_PQ + cb * 16384, 32 * cb, 0, sidx);
                        bulk_commit();
                    }
                    bulk_wait_read();
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}


// ------------------------------------------------------------- segments
// Segment-parallel state pass.  Each chunk maps the entering state affinely,
// h' = (Diag(gamma) + Phi) h + K~^T U, so a run of chunks (a segment j) does
// too: h_out = A_j h_in + b_j.  The chain kernel in segment mode 1 forms b_j
// (from a zero state) and A_j (from the identity, with no writes) for every
// segment at once; this kernel composes them in order, h_{j+1} = A_j h_j + b_j
// in fp32 from the wave's entering state h_0; the chain kernel in segment
// mode 3 then runs every segment from its h_j with outputs.  The columns v of
// the state evolve independently, so one CTA takes 16 of them for one
// (batch, head): thread (row d, 8 columns), h_j's 16 columns in shared
// memory, A_j there too (rows padded to 132 words: 16-byte aligned, two-way
// bank conflicts at most), the next A_j copied in (cp.async) while the
// current one is applied.
constexpr int SEGC_THREADS = 256;
constexpr int SEGC_COLS = 16;                  // state columns per CTA
constexpr int SEGC_LDA = 132;                  // row stride of A_j in shared memory (words)
constexpr uint32_t SEGC_SMEM = (2 * D * SEGC_LDA + D * SEGC_COLS) * sizeof(float);

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(SEGC_THREADS)
segment_combine_kernel(const ChunkParams p, const float* __restrict__ seg_b,
                       const float* __restrict__ seg_a) {
    extern __shared__ __align__(16) float smf[];
    float* As = smf;                          // A_j [2][D][SEGC_LDA]
    float* hs = smf + 2 * D * SEGC_LDA;       // h_j [D][SEGC_COLS]
    pdl_wait();                  // offsets and transitions are complete and visible
                                 // (no early launch of the output pass: its CTAs wait
                                 // for this grid and must not hold SMs it needs)
    constexpr int NG = D / SEGC_COLS;
    const int bh = blockIdx.x / NG, v0 = SEGC_COLS * (blockIdx.x % NG);
    const int S = p.nseg, t = threadIdx.x;
    const int d = t >> 1, c0 = 8 * (t & 1);
    // A_j -> buffer j & 1: 16 copies of 16 bytes a thread (rows of 32 chunks)
    auto fetch_a = [&](int j) {
        const float* src = seg_a + ((size_t)bh * S + j) * D * D;
        float* dst = As + (j & 1) * D * SEGC_LDA;
#pragma unroll
        for (int i = 0; i < D * D / 4 / SEGC_THREADS; ++i) {
            const int idx = t + SEGC_THREADS * i, row = idx >> 5, ch = idx & 31;
            cp_async16(dst + row * SEGC_LDA + 4 * ch, src + row * D + 4 * ch);
        }
        cp_async_commit();
    };
    if (S > 1) fetch_a(0);
    for (int idx = t; idx < D * SEGC_COLS; idx += SEGC_THREADS) {
        const int r = idx / SEGC_COLS, cc = idx % SEGC_COLS;
        hs[idx] = p.s0 ? __ldcg(p.s0 + (size_t)bh * D * D + r * D + v0 + cc) : 0.f;
    }
#pragma unroll 1
    for (int jj = 0; jj + 1 < S; ++jj) {
        const bool more = jj + 2 < S;
        if (more) fetch_a(jj + 1);
        float acc[8];
        const float* bsrc = seg_b + ((size_t)bh * S + jj) * D * D + d * D + v0 + c0;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = __ldcg(bsrc + e);
        if (more) cp_async_wait<1>();
        else cp_async_wait<0>();
        __syncthreads();         // A_j and h_j are in shared memory
        const float* arow = As + (jj & 1) * D * SEGC_LDA + d * SEGC_LDA;
#pragma unroll 8
        for (int dp = 0; dp < D; ++dp) {
            const float a = arow[dp];
            const float4 x0 = *reinterpret_cast<const float4*>(hs + dp * SEGC_COLS + c0);
            const float4 x1 = *reinterpret_cast<const float4*>(hs + dp * SEGC_COLS + c0 + 4);
            acc[0] = fmaf(a, x0.x, acc[0]);
            acc[1] = fmaf(a, x0.y, acc[1]);
            acc[2] = fmaf(a, x0.z, acc[2]);
            acc[3] = fmaf(a, x0.w, acc[3]);
            acc[4] = fmaf(a, x1.x, acc[4]);
            acc[5] = fmaf(a, x1.y, acc[5]);
            acc[6] = fmaf(a, x1.z, acc[6]);
            acc[7] = fmaf(a, x1.w, acc[7]);
        }
        __syncthreads();         // every thread is done with h_j and A_j's buffer
        float* dst = p.seg_h + ((size_t)bh * S + jj + 1) * D * D + d * D + v0 + c0;
        *reinterpret_cast<float4*>(hs + d * SEGC_COLS + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(hs + d * SEGC_COLS + c0 + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = acc[e];
    }
}

// Segments per (batch, head) for a wave of nchunks chunks: only when the
// heads leave most SMs idle (pass 1 runs two CTAs per segment, one per SM),
// with at least eight chunks a segment; 1 means the plain chain.
constexpr int kSegSMs = 148;
int segments_for(int nbh, int nchunks) {
    if (nbh > 16) return 1;
    const int S = std::min(kSegSMs / (2 * nbh), nchunks / 8);
    return std::max(S, 1);
}
size_t seg_bytes(int nbh, int NC) {
    const int S = segments_for(nbh, NC);
    return S > 1 ? (size_t)3 * nbh * S * D * D * sizeof(float) : 0;
}

bool make_maps(const ChunkParams& p, bool perdim, PrepMaps* m) {
    const uint64_t dims[3] = {(uint64_t)p.H * D, (uint64_t)p.T, (uint64_t)p.B};
    const uint64_t strides[2] = {(uint64_t)p.H * D * 2, (uint64_t)p.T * p.H * D * 2};
    const uint32_t box[3] = {64, 64, 1};
    bool ok = make_tmap_bf16(&m->q, p.q, 3, dims, strides, box) &&
              make_tmap_bf16(&m->k, p.k, 3, dims, strides, box) &&
              make_tmap_bf16(&m->v, p.v, 3, dims, strides, box);
    m->g = m->q;
    m->kw = m->k;
    if (ok && perdim) ok = make_tmap_bf16(&m->g, p.g, 3, dims, strides, box);
    if (ok && p.kw) ok = make_tmap_bf16(&m->kw, p.kw, 3, dims, strides, box);
    return ok;
}

// Item counters of the persistent prep, one per wave (at most one wave per
// chunk), at the end of the workspace.
size_t counter_bytes(int NC) { return ((size_t)NC * sizeof(unsigned) + 255) & ~(size_t)255; }

// Chunks per (batch, head) of one wave, for a workspace of `budget` bytes.
// Short sequences (up to 4 chunks) run as one wave.  Otherwise two image
// buffers alternate (plus the state carried between waves): the longest wave
// whose buffer fits the budget and WAVE_BYTES, at most half the chunks (so that
// a wave's chain overlaps the next wave's prep), and among such lengths the
// longest whose prep CTAs fill their last round of resident CTAs to at least
// 90 % (a nearly empty last round costs a whole CTA lifetime).  0 if even one
// chunk per wave does not fit.
int wave_chunks(int nbh, int NC, size_t budget) {
    if (budget < counter_bytes(NC)) return 0;
    budget -= counter_bytes(NC);
    const size_t per = (size_t)nbh * IMG_BYTES;                  // one chunk of every head
    const size_t carry = (size_t)nbh * D * D * sizeof(float);
    const bool fits_one = (size_t)NC * per <= budget;
    if (NC <= 4 && fits_one && (size_t)NC * per <= WAVE_BYTES) return NC;
    if (budget < 2 * per + carry) return fits_one ? NC : 0;
    long long cmax = std::min<long long>((long long)(WAVE_BYTES / per), (NC + 1) / 2);
    cmax = std::min<long long>(cmax, (long long)((budget - carry) / (2 * per)));
    if (cmax < 1) cmax = 1;
    for (long long c = cmax; c >= 1; --c) {
        const long long items = c * nbh;
        const long long rounds = (items + PREP_SLOTS - 1) / PREP_SLOTS;
        if (10 * items >= 9 * rounds * PREP_SLOTS) return (int)c;
    }
    return (int)cmax;
}

// Workspace of a forward whose waves are cw chunks long.
size_t workspace_for(int nbh, int NC, int cw) {
    const int nw = (NC + cw - 1) / cw;
    size_t bytes = (size_t)nbh * cw * IMG_BYTES * (nw > 1 ? 2 : 1);   // two alternating buffers
    if (nw > 1) bytes += (size_t)nbh * D * D * sizeof(float);           // state between waves
    return bytes + counter_bytes(NC);
}

// How a forward of NC chunks over nbh heads runs with ws_bytes of workspace:
// chunks per wave, waves, and whether the segment buffers are reserved.
struct Plan {
    int cw, nw, S_size;
    bool use_seg;
};
Plan plan_for(int B, int T, int H, int gate, size_t ws_bytes);

}  // namespace

size_t chunk_fwd_tc_capture_bytes(int B, int T, int H) {
    const int NC = (T + C - 1) / C;
    if (NC == 0 || B == 0 || H == 0) return 0;
    return (size_t)B * H * NC * IMG_BYTES + counter_bytes(NC);
}

cudaError_t launch_chunk_fwd_tc_capture(const ChunkParams& p0, int gate, size_t ws_bytes,
                                        float* h_all, cudaStream_t s, int* launches) {
    ChunkParams p = p0;
    p.h_all = h_all;
    p.nc_total = (p0.T + C - 1) / C;
    if (ws_bytes < chunk_fwd_tc_capture_bytes(p0.B, p0.T, p0.H)) return cudaErrorInvalidValue;
    return launch_chunk_fwd_tc(p, gate, ws_bytes, s, launches);
}

bool chunk_fwd_tc_supported(int Dk, int Dv, int gate) {
    return Dk == D && Dv == D && (gate == kGateNone || gate == kGateScalar || gate == kGatePerDim);
}

size_t chunk_fwd_tc_workspace_bytes(int B, int T, int H, int gate) {
    (void)gate;
    const int NC = (T + C - 1) / C;
    if (NC == 0 || B == 0 || H == 0) return 0;
    const int nbh = B * H;
    return workspace_for(nbh, NC, wave_chunks(nbh, NC, ~static_cast<size_t>(0))) + seg_bytes(nbh, NC);
}

namespace {
Plan plan_for(int B, int T, int H, int gate, size_t ws_bytes) {
    Plan pl{0, 0, 1, false};
    const int NC = (T + C - 1) / C;
    const int nbh = B * H;
    // segment buffers first, when the workspace holds them beside the least the
    // forward needs (the full-speed size does); then waves as long as the rest allows
    const size_t sbytes = seg_bytes(nbh, NC);
    pl.use_seg = sbytes > 0 && ws_bytes >= chunk_fwd_tc_workspace_min_bytes(B, T, H, gate) + sbytes;
    pl.cw = wave_chunks(nbh, NC, pl.use_seg ? ws_bytes - sbytes : ws_bytes);
    pl.nw = pl.cw > 0 ? (NC + pl.cw - 1) / pl.cw : 0;
    pl.S_size = pl.use_seg ? segments_for(nbh, NC) : 1;
    return pl;
}
// Segments of a wave of nchunks chunks (the launcher's rule).
int wave_segments(const Plan& pl, int nbh, int nchunks) {
    int Sw = pl.use_seg ? std::min(segments_for(nbh, nchunks), pl.S_size) : 1;
    if (Sw > 1) {
        const int L = (nchunks + Sw - 1) / Sw;
        Sw = (nchunks + L - 1) / L;
    }
    return Sw;
}
}  // namespace

void chunk_fwd_tc_plan(int B, int T, int H, int gate, size_t ws_bytes, int* waves,
                       int* chunks_per_wave, int* segments) {
    const Plan pl = plan_for(B, T, H, gate, ws_bytes);
    *waves = pl.nw;
    *chunks_per_wave = pl.cw;
    *segments = pl.cw > 0 ? wave_segments(pl, B * H, pl.cw) : 0;
}

size_t chunk_fwd_tc_workspace_min_bytes(int B, int T, int H, int gate) {
    (void)gate;
    const int NC = (T + C - 1) / C;
    if (NC == 0 || B == 0 || H == 0) return 0;
    const size_t per = (size_t)B * H * IMG_BYTES;
    const size_t two = 2 * per + (size_t)B * H * D * D * sizeof(float);
    return std::min((size_t)NC * per, two) + counter_bytes(NC);
}

cudaError_t launch_chunk_fwd_tc(const ChunkParams& p0, int gate, size_t ws_bytes, cudaStream_t s,
                                int* launches) {
    *launches = 0;
    const bool perdim = gate == kGatePerDim;
    PrepMaps maps;
    if (!make_maps(p0, perdim, &maps)) return cudaErrorInvalidValue;
    ChainMaps cmap0;
    memset(&cmap0, 0, sizeof(cmap0));
    {
        const uint64_t dims[3] = {(uint64_t)p0.H * D, (uint64_t)p0.T, (uint64_t)p0.B};
        const uint64_t strides[2] = {(uint64_t)p0.H * D * 2, (uint64_t)p0.T * p0.H * D * 2};
        const uint32_t box[3] = {64, 64, 1};
        if (!make_tmap_bf16(&cmap0.o, p0.o, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    // fp32 states [B*H][D rows][D columns], boxes of 128 rows x 32 columns
    auto state_map = [&](CUtensorMap* m, const float* base) {
        if (!base) return true;
        const uint64_t dims[3] = {(uint64_t)D, (uint64_t)D, (uint64_t)p0.B * p0.H};
        const uint64_t strides[2] = {(uint64_t)D * 4, (uint64_t)D * D * 4};
        const uint32_t box[3] = {32, 128, 1};
        return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 3, dims, strides, box);
    };
    using PrepFn = void (*)(const PrepMaps, const ChunkParams);
    const bool wk = p0.kw != nullptr;
    PrepFn prep = gate == kGateScalar ? (wk ? chunk_prep_kernel<kGateScalar, true>
                                            : chunk_prep_kernel<kGateScalar, false>)
                  : gate == kGatePerDim ? (wk ? chunk_prep_kernel<kGatePerDim, true>
                                              : chunk_prep_kernel<kGatePerDim, false>)
                                        : (wk ? chunk_prep_kernel<kGateNone, true>
                                              : chunk_prep_kernel<kGateNone, false>);
    const uint32_t prep_smem = P_SMEM;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem);
    if (e != cudaSuccess) return e;
    auto chain = gate == kGatePerDim ? chunk_chain_kernel<false> : chunk_chain_kernel<true>;
    e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CH_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(segment_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SEGC_SMEM);
    if (e != cudaSuccess) return e;
    const int NC = (p0.T + C - 1) / C;
    const int nbh = p0.B * p0.H;
    Plan pl = plan_for(p0.B, p0.T, p0.H, gate, ws_bytes);
    if (p0.h_all) {   // the backward's forward: one wave, every image kept, no segments
        pl.cw = NC;
        pl.nw = 1;
        pl.use_seg = false;
        pl.S_size = 1;
    }
    const bool use_seg = pl.use_seg;
    const int cw = pl.cw;
    if (cw < 1) return cudaErrorInvalidValue;
    const int nw = pl.nw;
    const size_t buf_bytes = (size_t)nbh * cw * IMG_BYTES;
    float* carry = nw > 1 ? reinterpret_cast<float*>(p0.ws + 2 * buf_bytes) : nullptr;
    unsigned* counters = reinterpret_cast<unsigned*>(
        p0.ws + workspace_for(nbh, NC, cw) - counter_bytes(NC));
    // persistent prep: two CTAs per SM take the wave's items from its counter
    static int sm_count[64] = {0};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!sm_count[dev]) {
        int c = 0;
        e = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        sm_count[dev] = c;
    }
    e = cudaMemsetAsync(counters, 0, (size_t)nw * sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    CUtensorMap m_sout, m_carry;
    memset(&m_sout, 0, sizeof(m_sout));
    memset(&m_carry, 0, sizeof(m_carry));
    if (!state_map(&m_sout, p0.s_out) || !state_map(&m_carry, carry)) return cudaErrorInvalidValue;
    // segment buffers after the counters: entering states [B*H][S][D][D], then
    // offsets and transitions [2][B*H][S][D][D]
    const int S_size = pl.S_size;
    float* seg_h = use_seg ? reinterpret_cast<float*>(p0.ws + workspace_for(nbh, NC, cw)) : nullptr;
    float* seg2 = use_seg ? seg_h + (size_t)nbh * S_size * D * D : nullptr;
    // Every launch but the first may start before its predecessor ends
    // (programmatic dependent launch); the kernels order themselves with
    // griddepcontrol (see chunk_prep_kernel and chunk_chain_kernel).
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    for (int w = 0; w < nw; ++w) {
        ChunkParams p = p0;
        p.ws = p0.ws + (size_t)(w & 1) * buf_bytes;
        p.cw = cw;
        p.ws_chunk = (int)IMG_BYTES;
        p.chunk0 = w * cw;
        p.nchunks = (w + 1 < nw) ? cw : NC - w * cw;
        p.s0 = (w == 0) ? p0.s0 : carry;
        p.s_out = (w + 1 == nw) ? p0.s_out : carry;
        p.counter = counters + w;
        const int items = nbh * p.nchunks;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(std::min(items, 2 * sm_count[dev]) + 1));
        cfg.blockDim = dim3(NPR);
        cfg.dynamicSmemBytes = prep_smem;
        cfg.stream = s;
        cfg.attrs = &pdl;
        cfg.numAttrs = w > 0 ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, prep, maps, p);
        if (e != cudaSuccess) return e;
        ++*launches;
        cfg.blockDim = dim3(CH_THREADS);
        cfg.dynamicSmemBytes = CH_SMEM;
        cfg.numAttrs = 1;
        ChainMaps cm = cmap0;
        cm.s_out = (w + 1 == nw) ? m_sout : m_carry;
        const int Sw = wave_segments(pl, nbh, p.nchunks);
        if (Sw > 1) {   // segment-parallel state pass: offsets and transitions,
                        // their composition, then every segment with outputs
            const int L = (p.nchunks + Sw - 1) / Sw;
            p.nseg = Sw;
            p.seg_len = L;
            p.seg_h = seg_h;
            {
                const uint64_t dims[3] = {(uint64_t)D, (uint64_t)D, (uint64_t)2 * nbh * Sw};
                const uint64_t strides[2] = {(uint64_t)D * 4, (uint64_t)D * D * 4};
                const uint32_t box[3] = {32, 128, 1};
                if (!make_tmap(&cm.seg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, seg2, 3, dims, strides, box))
                    return cudaErrorInvalidValue;
            }
            p.seg_mode = 1;
            cfg.gridDim = dim3((unsigned)(2 * nbh * Sw));
            e = cudaLaunchKernelEx(&cfg, chain, cm, p);
            if (e != cudaSuccess) return e;
            ++*launches;
            cudaLaunchConfig_t cc = cfg;
            cc.gridDim = dim3((unsigned)(nbh * (D / SEGC_COLS)));
            cc.blockDim = dim3(SEGC_THREADS);
            cc.dynamicSmemBytes = SEGC_SMEM;
            const float* sb_ = seg2;
            const float* sa_ = seg2 + (size_t)nbh * Sw * D * D;
            e = cudaLaunchKernelEx(&cc, segment_combine_kernel, p, sb_, sa_);
            if (e != cudaSuccess) return e;
            ++*launches;
            p.seg_mode = 3;
            cfg.gridDim = dim3((unsigned)(nbh * Sw));
        } else {
            p.seg_mode = 0;
            cfg.gridDim = dim3((unsigned)nbh);
        }
        e = cudaLaunchKernelEx(&cfg, chain, cm, p);
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;   // every launch's own status was checked above
}

}  // namespace gdn
