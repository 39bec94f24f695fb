// The Mix-FFN of the Linear DiT block ("Sana: Efficient High-Resolution Image
// Synthesis with Linear Diffusion Transformers", section 2.2: an inverted residual
// block, a 3x3 depthwise convolution and a GLU in place of the MLP FFN; section
// 2.3: the convolution's zero padding carries position; "SANA 1.5", section
// "Model architecture": C = 2240, FFN width F = 5600).  Tokens n = y * Ws + x of a
// row-major (Hs, Ws) grid:
//   U  = X W1 + b1                    gemm_bias_bf16_2sm (1x1 expand, C -> 2F)
//   Hg = Cv[:, :F] * gate(Cv[:, F:]), dwconv3x3_glu      (depthwise 3x3 with zero
//        Cv = dwconv3x3(U) + bdw                          padding, then the GLU)
//   Y  = Hg W2 + b2                   gemm_bias_bf16_2sm (1x1 project, F -> C)
// U and Hg are stored in bf16; every sum accumulates in fp32.
//
// gemm_bias_bf16_2sm: D[M][Nc] = A[M][K] W[K][Nc] (+ bias) on the sm_100a tensor
//   cores, each UMMA spread over a pair of SMs (256 x 256 tiles; see below).
//   Persistent: pair p takes tiles p, p + pairs, ... in groups of 2 row-pair blocks
//   with the row block fastest inside a group, so concurrent pairs share A rows and
//   a band of W columns through L2.  Warp 0 is the TMA producer (7-stage ring of
//   the CTA's A 128 x 64 k, K-major, and its W 64 k x 128 n, MN-major, both
//   128-byte swizzled), warp 1 of the leader CTA issues the UMMAs into one of two
//   TMEM accumulators, warps 2-9 of both CTAs drain the other (bias, bf16,
//   stores), so a tile's epilogue overlaps the next tile's main loop.
// dwconv3x3_glu: CTA (channel chunk, column strip, batch) marches down the grid
//   rows of a 32-token strip for 32 value channels and the 32 matching gate
//   channels.  An 8-row TMA ring brings in each input row once, with one halo
//   token on each side (coordinates outside the grid read as zeros: the padding);
//   each thread keeps three rolling output rows in registers, so input row r is
//   added to outputs r + 1, r and r - 1 with kernel rows 0, 1 and 2, and output
//   r - 1 is complete after input r.
#pragma once

#include "f32x2.cuh"
#include "sana_common.cuh"
#include "sm100_pair.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

enum GateKind : int { kGateSigmoid = 0, kGateSilu = 1 };

__device__ __forceinline__ void tma_load_4d_u(void* dst, const CUtensorMap* m, uint64_t* bar,
                                              int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// ============================================================================ GEMM
struct GemmArgs {
    const float* bias;   // [Nc] or nullptr
    bf16* d;             // [M][Nc] row-major
    int64_t M;
    int Nc, K;
    int mb, nb;          // 128-row blocks along M, 256-column blocks along Nc
};

// ============================================================================ GEMM, 2 SMs
// The same D = A W (+ bias) with the UMMA spread over a pair of SMs (a cluster of
// two CTAs, tcgen05 cta_group::2): one instruction computes a 256 x 256 x 16 tile
// step, CTA r of the pair supplying rows [128 r, 128 r + 128) of the A tile and
// columns [128 r, 128 r + 128) of the W tile from its own shared memory, and
// receiving rows [128 r, + 128) x all 256 columns of the product in its own TMEM.
// Each SM thus streams 32 KB of operands per 64-deep k step instead of 48 KB for
// the same tensor work: the single-SM kernel is bound by that stream from L2.
//
// Hand-offs: both CTAs' TMA loads (unicast, each into its own shared memory)
// complete on the leader CTA's `full` barrier (the cta_group::2 form of the load),
// which the leader's producer arms with the bytes of both halves; only the leader
// issues UMMAs, and its commits arrive on `empty` and `accfull` in both CTAs at
// once (the commit's CTA mask); both CTAs' epilogue warps arrive on the leader's
// `accempty`.  (Passing the leader's phases on to the peer by remote arrives
// instead, with no mask on the commit, measured half the speed: a stage's round
// trip then carries two more hand-offs.)
namespace g2 {
constexpr int kBM = 128;                        // rows per CTA (the pair: 256)
constexpr int kBN = 256;                        // columns per tile (128 per CTA's W half)
constexpr int kBK = 64;
constexpr int kABytes = kBM * 128;              // 16 KB
constexpr int kWBox = kBK * 128;                // 8 KB: 64 k rows x 64 n
constexpr int kWBoxes = 2;                      // this CTA's 128 columns
constexpr int kStageBytes = kABytes + kWBoxes * kWBox;   // 32 KB
constexpr int kStages = 7;
constexpr int kTmemCols = 2 * kBN;              // two accumulators
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
static_assert(kSmemBytes <= 232448, "shared memory");
constexpr int kGroupPairs = 2;                  // row-pair blocks per raster group
}  // namespace g2

// Tile t -> (row-pair block, column block), grouped as gemm_tile does.
__device__ __forceinline__ void gemm_tile2(int64_t t, int mb2, int nb, int& mblk, int& nblk) {
    const int64_t per_group = (int64_t)g2::kGroupPairs * nb;
    const int64_t grp = t / per_group, local = t % per_group;
    const int rows = (int)min((int64_t)g2::kGroupPairs, mb2 - grp * g2::kGroupPairs);
    nblk = (int)(local / rows);
    mblk = (int)(grp * g2::kGroupPairs + local % rows);
}

__global__ void __launch_bounds__(g2::kThreads, 1)
gemm_bias_bf16_2sm(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_w, const GemmArgs a)
{
    using namespace g2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint64_t* full = (uint64_t*)(stages + kStages * kStageBytes);   // used in the leader
    uint64_t* empty = full + kStages;
    uint64_t* accfull = empty + kStages;         // [2]
    uint64_t* accempty = accfull + 2;            // [2], used in the leader
    uint64_t* drained = accempty + 2;
    uint32_t* tmem_slot = (uint32_t*)(drained + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = blockIdx.x & 1;        // rank in the cluster of two
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int mb2 = (int)((a.M + 2 * kBM - 1) / (2 * kBM));
    const int64_t tiles = (int64_t)mb2 * a.nb;
    const int ksteps = (a.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 2 * kEpiWarps);
        }
        mbar_init(drained, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_w);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();                            // both CTAs' barriers are initialised
    cluster_wait();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int64_t step = 0;
            for (int64_t t = pair; t < tiles && ok; t += npairs) {
                int mblk, nblk;
                gemm_tile2(t, mb2, a.nb, mblk, nblk);
                const int m0 = mblk * 2 * kBM + (int)rank * kBM;
                const int n0 = nblk * kBN + (int)rank * (kBN / 2);
                for (int kk = 0; kk < ksteps; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    if (step >= kStages) {
                        ok = mbar_wait_spin(&empty[st], (uint32_t)((step / kStages) - 1) & 1, 621);
                        if (!ok) break;
                    }
                    uint8_t* sb = stages + st * kStageBytes;
                    const uint32_t fb = map_shared_rank(smem_u32(&full[st]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[st], 2 * kStageBytes);
                    tma_load_2d_pair(sb, &tmap_a, fb, kk * kBK, m0);
#pragma unroll
                    for (int j = 0; j < kWBoxes; ++j)
                        tma_load_2d_pair(sb + kABytes + j * kWBox, &tmap_w, fb, n0 + 64 * j,
                                         kk * kBK);
                }
            }
            // Before the CTA may exit, every slot's last load must have been consumed.
            const int64_t n = step;
            for (int64_t s2 = n - kStages > 0 ? n - kStages : 0; s2 < n && ok; ++s2)
                ok = mbar_wait(&empty[s2 % kStages], (uint32_t)(s2 / kStages) & 1, 622);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer (the leader's lane 0)
        if (leader && lane == 0) {
            const uint32_t idesc = make_idesc_bf16(2 * kBM, kBN, false, true);
            int64_t step = 0;
            int lt = 0;
            for (int64_t t = pair; t < tiles && ok; t += npairs, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2) ok = mbar_wait(&accempty[buf], (uint32_t)((lt >> 1) - 1) & 1, 624);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t acc = tmem + buf * kBN;
                for (int kk = 0; kk < ksteps; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    ok = mbar_wait_spin(&full[st], (uint32_t)(step / kStages) & 1, 625);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t ab = smem_u32(stages + st * kStageBytes);
                    const uint32_t wb = ab + kABytes;
#pragma unroll
                    for (int k4 = 0; k4 < kBK / 16; ++k4) {
                        const uint64_t ad = make_smem_desc(ab + k4 * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_smem_desc(wb + k4 * 16 * 128, kWBox, 1024,
                                                           kSwizzle128B);
                        umma_bf16_pair(acc, ad, bd, idesc, kk > 0 || k4 > 0);
                    }
                    umma_commit_both(&empty[st]);
                }
                if (!ok) break;
                umma_commit_both(&accfull[buf]);
            }
            umma_commit_pair(drained);
            mbar_wait(drained, 0, 626);
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs: own rows)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        int lt = 0;
        for (int64_t t = pair; t < tiles && ok; t += npairs, ++lt) {
            const int buf = lt & 1;
            ok = mbar_wait(&accfull[buf], (uint32_t)(lt >> 1) & 1, 627);
            if (!ok) break;
            tc_fence_after_sync();
            int mblk, nblk;
            gemm_tile2(t, mb2, a.nb, mblk, nblk);
            const int64_t row = (int64_t)mblk * 2 * kBM + (int)rank * kBM + 32 * q + lane;
            const int n0 = nblk * kBN;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const int col = half * 128 + c * 32;
                float v[32];
                const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + buf * kBN + col;
                tmem_ld16(ta, v);
                tmem_ld16(ta + 16, v + 16);
                tmem_wait_ld();
                const int n = n0 + col;
                if (n >= a.Nc) break;
                if (a.bias) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (n + i < a.Nc) v[i] += __ldg(a.bias + n + i);
                }
                if (row < a.M) {
                    bf16* dst = a.d + row * a.Nc + n;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8)
                        if (n + 8 * g8 < a.Nc) store8(dst + 8 * g8, v + 8 * g8);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(map_shared_rank(smem_u32(&accempty[buf]), 0));
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_arrive();                            // both CTAs are done with the TMEM
    cluster_wait();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ============================================================================ dwconv + GLU
namespace dw {
constexpr int kTX = 32;                         // output tokens per CTA along a grid row
constexpr int kCh = 32;                         // value channels per CTA (+ 32 gate channels)
constexpr int kBoxTok = kTX + 2;                // one halo token on each side
constexpr int kTokBytes = kCh * 2;              // 64 B of one token in a ring row
constexpr int kRowBytes = kBoxTok * kTokBytes;  // 2176 B
constexpr int kSlotBytes = 2 * kRowBytes;       // value row + gate row
constexpr int kSlots = 8;                       // input rows in flight
constexpr int kThreads = 256;                   // (token x: 32) x (4-channel group: 8)
}  // namespace dw

// Output row of 4 value + 4 gate channels: pairs 0, 1 value, 2, 3 gate.
// GLU with the gate sigmoid(z) = 1 / (1 + e^-z) from __expf and __fdividef (a
// few fp32 ulps; e^-z = inf gives 0), then bf16 rounding and one 8-byte store.
template <int kGate>
__device__ __forceinline__ void glu_store4(bf16* p, const uint64_t* acc) {
    float a[4], z[4];
    unpack2(acc[0], a[0], a[1]);
    unpack2(acc[1], a[2], a[3]);
    unpack2(acc[2], z[0], z[1]);
    unpack2(acc[3], z[2], z[3]);
    float o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float sg = __fdividef(1.f, 1.f + __expf(-z[c]));
        o[c] = a[c] * (kGate == kGateSigmoid ? sg : z[c] * sg);
    }
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
}

// u: (B, Hs, Ws, 2F) bf16 seen by TMA as 4-D (2F, Ws, Hs, B), boxes of 32 channels
// x 34 tokens x 1 row x 1 batch.  wdw [2F][3][3] fp32, bdw [2F] fp32 or nullptr,
// h (B, Hs*Ws, F) bf16.  grid (ceil(F / 32), ceil(Ws / 32), B).  F % 8 == 0.
// Thread (x, cg) owns value channels j0..j0+3 (j0 = c0 + 4 cg) and the matching gate
// channels of grid column x0 + x; output row y lives in the accumulator set
// acc[y % 3] (4 packed pairs), so the march needs no register moves.
template <int kGate>
__global__ void __launch_bounds__(dw::kThreads, 2)
dwconv3x3_glu(const __grid_constant__ CUtensorMap tmap_u, const float* __restrict__ wdw,
              const float* __restrict__ bdw, bf16* __restrict__ h, int Hs, int Ws, int F)
{
    using namespace dw;
    __shared__ __align__(128) uint8_t ring[kSlots][kSlotBytes];
    __shared__ __align__(8) uint64_t full[kSlots];
    const int c0 = blockIdx.x * kCh, x0 = blockIdx.y * kTX, b = blockIdx.z;
    const int t = threadIdx.x, cg = t & 7, x = t >> 3;
    const int j0 = c0 + 4 * cg;                        // first value channel of the thread
    const bool chan_live = j0 < F;                     // F % 4 == 0: all 4 or none
    const bool live = chan_live && x0 + x < Ws;

    if (t == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
        prefetch_tmap(&tmap_u);
    }
    __syncthreads();
    int issued = 0;                                    // rows issued (thread 0)
    auto issue = [&]() {
        const int s = issued % kSlots;
        mbar_arrive_expect_tx(&full[s], kSlotBytes);
        tma_load_4d_u(ring[s], &tmap_u, &full[s], c0, x0 - 1, issued, b);
        tma_load_4d_u(ring[s] + kRowBytes, &tmap_u, &full[s], F + c0, x0 - 1, issued, b);
        ++issued;
    };
    if (t == 0)
        while (issued < kSlots && issued < Hs) issue();

    // w2[k][p]: tap k (= 3 i + j) of channel pair p (0, 1 value; 2, 3 gate)
    uint64_t w2[9][4], bias2[4];
    {
        const int jv = chan_live ? j0 : 0, jg = chan_live ? F + j0 : 0;
        const float* wv = wdw + (int64_t)jv * 9;
        const float* wg = wdw + (int64_t)jg * 9;
#pragma unroll
        for (int k = 0; k < 9; ++k) {
            w2[k][0] = pack2(__ldg(wv + k), __ldg(wv + 9 + k));
            w2[k][1] = pack2(__ldg(wv + 18 + k), __ldg(wv + 27 + k));
            w2[k][2] = pack2(__ldg(wg + k), __ldg(wg + 9 + k));
            w2[k][3] = pack2(__ldg(wg + 18 + k), __ldg(wg + 27 + k));
        }
        bias2[0] = bdw ? pack2(__ldg(bdw + jv), __ldg(bdw + jv + 1)) : 0ull;
        bias2[1] = bdw ? pack2(__ldg(bdw + jv + 2), __ldg(bdw + jv + 3)) : 0ull;
        bias2[2] = bdw ? pack2(__ldg(bdw + jg), __ldg(bdw + jg + 1)) : 0ull;
        bias2[3] = bdw ? pack2(__ldg(bdw + jg + 2), __ldg(bdw + jg + 3)) : 0ull;
    }
    // Output row y accumulates in A[y % 3].  Its first term (kernel row 0, input
    // row y - 1) starts from the bias; output 0 has no such term and starts there.
    uint64_t A0[4], A1[4], A2[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) A0[p] = A1[p] = A2[p] = bias2[p];

    bool ok = true;
    int waited = 0;                                    // rows this thread has waited for
    const int roff = x * kTokBytes + cg * 8;
    const int64_t row_pitch = (int64_t)Ws * F;                 // elements between grid rows
    bf16* out = h + (((int64_t)b * Hs) * Ws + x0 + x) * F + j0;   // output row 0

    // input row r: up = output r + 1 (kernel row 0), mid = output r (row 1),
    // dn = output r - 1 (row 2), complete after this row
    auto row = [&](int r, uint64_t (&up)[4], uint64_t (&mid)[4], uint64_t (&dn)[4]) {
        const int s = r % kSlots;
        if (ok) ok = mbar_wait(&full[s], (uint32_t)(r / kSlots) & 1, 701);
        if (ok) waited = r + 1;
        const uint8_t* rv = ring[s] + roff;
#pragma unroll
        for (int dx = 0; dx < 3; ++dx) {
            const uint2 pv = *reinterpret_cast<const uint2*>(rv + dx * kTokBytes);
            const uint2 pg = *reinterpret_cast<const uint2*>(rv + kRowBytes + dx * kTokBytes);
            const uint64_t in[4] = {bf16x2_to_f32x2(pv.x), bf16x2_to_f32x2(pv.y),
                                    bf16x2_to_f32x2(pg.x), bf16x2_to_f32x2(pg.y)};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                up[p] = fma2(w2[dx][p], in[p], dx == 0 ? bias2[p] : up[p]);   // a new row
                mid[p] = fma2(w2[3 + dx][p], in[p], mid[p]);
                dn[p] = fma2(w2[6 + dx][p], in[p], dn[p]);
            }
        }
        __syncthreads();                               // slot s is free
        if (t == 0 && ok && issued < Hs) {
            fence_proxy_async_smem();
            issue();
        }
        if (r >= 1) {
            if (live) glu_store4<kGate>(out, dn);
            out += row_pitch;
        }
    };
    for (int r = 0; r < Hs; r += 3) {
        row(r, A1, A0, A2);
        if (r + 1 < Hs) row(r + 1, A2, A1, A0);
        if (r + 2 < Hs) row(r + 2, A0, A2, A1);
    }
    if (Hs >= 1 && live) {               // out now points at output row Hs - 1
        const uint64_t* last = (Hs - 1) % 3 == 0 ? A0 : ((Hs - 1) % 3 == 1 ? A1 : A2);
        glu_store4<kGate>(out, last);
    }
    // after a timeout, let the copies already issued land before the CTA exits
    if (t == 0 && !ok)
        for (int r = waited; r < issued; ++r)
            mbar_wait(&full[r % kSlots], (uint32_t)(r / kSlots) & 1, 702);
}

}  // namespace sana
