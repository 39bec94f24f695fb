// Tensor-core (tcgen05 + TMA) kernels for the two passes of Eq. (1), "Sana:
// Efficient High-Resolution Image Synthesis with Linear Diffusion Transformers",
// section 2.1, with the per-head QK-RMSNorm of "SANA 1.5 ...", section "Model
// architecture" (QK Norm bullet).  bf16 inputs and outputs, fp32 accumulation.
//
// Both passes are HBM-bound (16.5 flop per byte); the D x (D+1) contractions go
// to the tensor cores only because CUDA-core FMAs cannot keep up with HBM here.
//
// Pass 1, kv_partial_tc.  CTA (s, g, b) reduces the tokens of split s for the
// head group g = 4 heads (128 channels) of batch b:
//     D[(h,d), (h',e)] = sum_t phi(K)[t,(h,d)] V[t,(h',e)]        (UMMA M=128, N=128)
//     D[(h,d), 128]    = sum_t phi(K)[t,(h,d)]                    (UMMA N=64, ones)
// and keeps the diagonal blocks h == h'.  K and V tiles arrive by TMA with the
// 128-byte swizzle, [token][channel]; the workers rewrite the K tile in place
// with phi(K) = ReLU(g * k / rms(k)), which turns it into the MN-major A operand;
// the V tile is already the MN-major B operand.
//
// Pass 2, apply_tc.  CTA (c, p, b) handles token tiles of 128 for the head pair
// p (64 channels) of batch b.  The workers build the B operand per head from
// the fp32 state (n = value column e or the normaliser, k = d; a bf16 hi part and
// a bf16 lo part so the state keeps ~16 mantissa bits), rewrite each Q tile in
// place with phi(Q) (the K-major A operand), the MMA warp computes
//     D[t, e] = sum_d phi(Q)[t,d] S[d,e],  e < 32;   D[t, 32] = sum_d phi(Q)[t,d] S[d,32]
// (UMMA M=128, N=48, K=16 x 2 x {hi, lo}), and the workers read D from TMEM,
// form O = D[:, :32] / (D[:, 32] + eps), write O over the tile and TMA-store it.
//
// Warp roles (192 threads): warp 0 issues TMA, warp 1 owns TMEM and issues UMMA,
// warps 2..5 transform operands and run the epilogue; warp w reads TMEM lanes
// 32 * (w % 4) .. + 31.
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"

namespace sana {

namespace tc1 {
constexpr int kStageTok = 64;                      // tokens per pipeline stage
constexpr int kGroupHeads = 4;                     // heads per CTA (UMMA M = 128)
constexpr int kBoxBytes = kStageTok * 128;         // one TMA box: 64 tokens x 64 channels
constexpr int kStageBytes = 4 * kBoxBytes;         // K box 0, K box 1, V box 0, V box 1
constexpr int kStages = 3;
constexpr int kOnesBytes = 16 * 128;               // 16 token rows x 64 columns
constexpr int kTmemCols = 256;                     // 128 value columns + 64 normaliser columns
constexpr int kThreads = 192;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kOnesBytes + 1024;
}  // namespace tc1

namespace tc2 {
constexpr int kTileTok = 128;                      // UMMA M
constexpr int kPairHeads = 2;                      // 64 channels = one swizzled row
constexpr int kTileBytes = kTileTok * 128;         // 16 KB
constexpr int kStages = 4;
constexpr int kN = 48;                             // 32 value columns, normaliser, padding
constexpr int kBopBytes = kN * 128;                // per head: rows n, [hi d0..31 | lo d0..31]
constexpr int kBufCols = kPairHeads * kN;          // 96 TMEM columns per tile
constexpr int kTmemCols = 256;                     // two tile buffers
constexpr int kThreads = 192;
constexpr int kSmemBytes = 1024 + kStages * kTileBytes + kPairHeads * kBopBytes + 1024;
}  // namespace tc2

// Apply phi = ReLU(g * x * rsqrt(mean(x^2) + eps)) (or ReLU(x) with the norm off)
// to 32 values held as 4 swizzled 16-byte chunks of row `row` starting at chunk
// `chunk0`, in place.  zero: write zeros instead (rows past N, heads past H).
__device__ __forceinline__ void phi_inplace_sw128(uint8_t* tile, int row, int chunk0,
                                                  const float* __restrict__ g, float eps,
                                                  bool norm, bool zero) {
    uint4 u[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
        u[c] = *reinterpret_cast<const uint4*>(tile + sw128_offset(row, chunk0 + c));
    float x[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        x[8 * c + 0] = bf16lo(u[c].x); x[8 * c + 1] = bf16hi(u[c].x);
        x[8 * c + 2] = bf16lo(u[c].y); x[8 * c + 3] = bf16hi(u[c].y);
        x[8 * c + 4] = bf16lo(u[c].z); x[8 * c + 5] = bf16hi(u[c].z);
        x[8 * c + 6] = bf16lo(u[c].w); x[8 * c + 7] = bf16hi(u[c].w);
    }
    if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(x[i], x[i], ss);
        const float r = rsqrtf(ss * (1.f / kD) + eps);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = fmaxf(g[i] * (x[i] * r), 0.f);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = fmaxf(x[i], 0.f);
    }
    if (zero) {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4*>(tile + sw128_offset(row, chunk0 + c)) = w;
    }
}

// ============================================================================ pass 1
// grid (S, ceil(H/4), B), 192 threads, tc1::kSmemBytes dynamic shared memory.
// part[((b*H + h)*S + s)][d][D+1]: the split's partial state.
__global__ void __launch_bounds__(tc1::kThreads, 2)
kv_partial_tc(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
              const float* __restrict__ gk, float* __restrict__ part, int N, int H, int S,
              int tps, float eps, int norm)
{
    using namespace tc1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* stages = smem;
    uint8_t* ones = smem + kStages * kStageBytes;
    uint64_t* full = (uint64_t*)(ones + kOnesBytes);
    uint64_t* aready = full + kStages;
    uint64_t* empty = aready + kStages;
    uint64_t* accdone = empty + kStages;
    uint64_t* drain = accdone + 1;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    float* sg = (float*)(tmem_slot + 4);            // 128 gains of the head group

    const int s = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = s * tps;
    const int n1 = min(N, n0 + tps);
    const int nst = (n1 - n0 + kStageTok - 1) / kStageTok;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], 128);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accdone, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    // the constant normaliser operand: column 0 of every row is 1.0
    for (int i = threadIdx.x; i < kOnesBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(ones)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
        const int h = grp * kGroupHeads + i / kD;
        sg[i] = (norm && h < H) ? gk[(size_t)h * kD + (i % kD)] : 1.f;
    }
    __syncthreads();
    if (threadIdx.x < 16) {
        const int r = threadIdx.x;
        *reinterpret_cast<uint16_t*>(ones + sw128_offset(r, 0)) = 0x3F80;   // bf16 1.0
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued[kStages] = {0, 0, 0};
            for (int t = 0; t < nst && ok; ++t) {
                const int st = t % kStages;
                if (t >= kStages) ok = mbar_wait(&empty[st], ((t / kStages) - 1) & 1, 101);
                if (!ok) break;
                uint8_t* sb = stages + st * kStageBytes;
                mbar_arrive_expect_tx(&full[st], kStageBytes);
                const int x = grp * 128, y = n0 + t * kStageTok;
                tma_load_3d(sb, &tmap_k, &full[st], x, y, b);
                tma_load_3d(sb + kBoxBytes, &tmap_k, &full[st], x + 64, y, b);
                tma_load_3d(sb + 2 * kBoxBytes, &tmap_v, &full[st], x, y, b);
                tma_load_3d(sb + 3 * kBoxBytes, &tmap_v, &full[st], x + 64, y, b);
                issued[st] = t + 1;
            }
            if (!ok) {   // let every issued copy land before the CTA can exit
                for (int st = 0; st < kStages; ++st)
                    if (issued[st]) mbar_wait(&full[st], ((issued[st] - 1) / kStages) & 1, 102);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (lane == 0) {
            const uint32_t idesc_v = make_idesc_bf16(128, 128, true, true);
            const uint32_t idesc_1 = make_idesc_bf16(128, 64, true, true);
            const uint64_t ones_desc = make_smem_desc(smem_u32(ones), kBoxBytes, 1024, kSwizzle128B);
            for (int t = 0; t < nst && ok; ++t) {
                const int st = t % kStages;
                ok = mbar_wait(&aready[st], (t / kStages) & 1, 103);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t kb = smem_u32(stages + st * kStageBytes);
                const uint32_t vb = kb + 2 * kBoxBytes;
#pragma unroll
                for (int kk = 0; kk < kStageTok / 16; ++kk) {
                    const uint64_t a = make_smem_desc(kb + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
                    const uint64_t bv = make_smem_desc(vb + kk * 2048, kBoxBytes, 1024, kSwizzle128B);
                    const bool acc = (t > 0) || (kk > 0);
                    umma_bf16(tmem, a, bv, idesc_v, acc);
                    umma_bf16(tmem + 128, a, ones_desc, idesc_1, acc);
                }
                umma_commit(&empty[st]);
            }
            umma_commit(ok ? accdone : drain);
            if (!ok) mbar_wait(drain, 0, 104);
        }
    } else {
        // ------------------------------------------------ operand transform + epilogue
        const int wt = threadIdx.x - 64;                 // 0..127
        const int row = wt & 63, box = wt >> 6;          // token row, channel box (2 heads)
        for (int t = 0; t < nst && ok; ++t) {
            const int st = t % kStages;
            ok = mbar_wait(&full[st], (t / kStages) & 1, 105);
            if (!ok) break;
            uint8_t* kt = stages + st * kStageBytes + box * kBoxBytes;
            const bool row_live = n0 + t * kStageTok + row < n1;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int hl = box * 2 + jj;             // head within the group
                const bool live = row_live && (grp * kGroupHeads + hl < H);
                phi_inplace_sw128(kt, row, jj * 4, sg + hl * kD, eps, norm != 0, !live);
            }
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
        }
        if (ok) ok = mbar_wait(accdone, 0, 106);
        if (ok) {
            tc_fence_after_sync();
            const int q = warp & 3;                      // TMEM lane quadrant = head in group
            const int h = grp * kGroupHeads + q;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16);
            float v[32], ks;
            tmem_ld16(ta + 32 * q, v);
            tmem_ld16(ta + 32 * q + 16, v + 16);
            tmem_ld1(ta + 128, &ks);
            tmem_wait_ld();
            if (h < H) {
                float* o = part + (((size_t)b * H + h) * S + s) * kStateFloats + lane * kDP;
#pragma unroll
                for (int e = 0; e < kD; ++e) o[e] = v[e];
                o[kD] = ks;
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ============================================================================ pass 2
// grid (ceil(tiles / tiles_per_cta), ceil(H/2), B), 192 threads, tc2::kSmemBytes.
__global__ void __launch_bounds__(tc2::kThreads, 2)
apply_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_o,
         const float* __restrict__ kv, const float* __restrict__ gq, int N, int H,
         int tiles_per_cta, float eps, int norm)
{
    using namespace tc2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* stages = smem;
    uint8_t* bop = smem + kStages * kTileBytes;
    uint64_t* full = (uint64_t*)(bop + kPairHeads * kBopBytes);
    uint64_t* aready = full + kStages;
    uint64_t* mmadone = aready + kStages;
    uint64_t* empty = mmadone + kStages;
    uint64_t* tfree = empty + kStages;
    uint64_t* bready = tfree + 2;
    uint64_t* drain = bready + 1;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    float* sg = (float*)(tmem_slot + 4);             // 64 gains of the head pair

    const int pair = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (N + kTileTok - 1) / kTileTok;
    const int tile0 = blockIdx.x * tiles_per_cta;
    const int nt = min(tiles_per_cta, n_tiles - tile0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], 128);
            mbar_init(&mmadone[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(&tfree[0], 128);
        mbar_init(&tfree[1], 128);
        mbar_init(bready, 128);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_o);
    }
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
        const int h = pair * kPairHeads + i / kD;
        sg[i] = (norm && h < H) ? gq[(size_t)h * kD + (i % kD)] : 1.f;
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = nt > 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && ok) {
            int issued[kStages] = {0, 0, 0, 0};
            for (int t = 0; t < nt && ok; ++t) {
                const int st = t % kStages;
                if (t >= kStages) ok = mbar_wait(&empty[st], ((t / kStages) - 1) & 1, 201);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[st], kTileBytes);
                tma_load_3d(stages + st * kTileBytes, &tmap_q, &full[st], pair * 64,
                            (tile0 + t) * kTileTok, b);
                issued[st] = t + 1;
            }
            if (!ok) {
                for (int st = 0; st < kStages; ++st)
                    if (issued[st]) mbar_wait(&full[st], ((issued[st] - 1) / kStages) & 1, 202);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (lane == 0 && ok) {
            const uint32_t idesc = make_idesc_bf16(128, kN, false, false);
            ok = mbar_wait(bready, 0, 203);
            for (int t = 0; t < nt && ok; ++t) {
                const int st = t % kStages, buf = t & 1;
                ok = mbar_wait(&aready[st], (t / kStages) & 1, 204);
                if (ok && t >= 2) ok = mbar_wait(&tfree[buf], ((t >> 1) - 1) & 1, 205);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t ab = smem_u32(stages + st * kTileBytes);
#pragma unroll
                for (int j = 0; j < kPairHeads; ++j) {
                    const uint32_t d = tmem + buf * kBufCols + j * kN;
                    const uint32_t bb = smem_u32(bop + j * kBopBytes);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t a = make_smem_desc(ab + j * 64 + kk * 32, 16, 1024,
                                                          kSwizzle128B);
                        const uint64_t hi = make_smem_desc(bb + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t lo = make_smem_desc(bb + 64 + kk * 32, 16, 1024,
                                                           kSwizzle128B);
                        umma_bf16(d, a, hi, idesc, kk > 0);
                        umma_bf16(d, a, lo, idesc, true);
                    }
                }
                umma_commit(&mmadone[st]);
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 206);
        }
    } else {
        // ------------------------------------------------ transform + epilogue
        const int wt = threadIdx.x - 64;                 // 0..127
        const int q = warp & 3;                          // TMEM lane quadrant
        const int row = 32 * q + lane;                   // token row of the tile
        // B operand from the fp32 state: rows n (value column e, normaliser at 32,
        // zero padding above), 16-byte chunks c: hi of d = 8c..8c+7 for c < 4, lo for c >= 4.
        for (int i = wt; i < kPairHeads * kN * 8; i += 128) {
            const int j = i / (kN * 8), rem = i % (kN * 8), n = rem >> 3, c = rem & 7;
            const int h = pair * kPairHeads + j;
            float vals[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int dd = (c & 3) * 8 + u;
                float x = 0.f;
                if (h < H && n <= kD) x = kv[((size_t)b * H + h) * kStateFloats + dd * kDP + n];
                const float hi = __bfloat162float(__float2bfloat16_rn(x));
                vals[u] = (c < 4) ? hi : (x - hi);
            }
            uint4 w;
            w.x = pack_bf16x2(vals[0], vals[1]);
            w.y = pack_bf16x2(vals[2], vals[3]);
            w.z = pack_bf16x2(vals[4], vals[5]);
            w.w = pack_bf16x2(vals[6], vals[7]);
            *reinterpret_cast<uint4*>(bop + j * kBopBytes + sw128_offset(n, c)) = w;
        }
        fence_proxy_async_smem();
        mbar_arrive(bready);

        auto transform = [&](int t) -> bool {
            const int st = t % kStages;
            if (!mbar_wait(&full[st], (t / kStages) & 1, 207)) return false;
            uint8_t* tile = stages + st * kTileBytes;
            const bool row_live = (tile0 + t) * kTileTok + row < N;
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                const bool live = row_live && (pair * kPairHeads + j < H);
                phi_inplace_sw128(tile, row, j * 4, sg + j * kD, eps, norm != 0, !live);
            }
            fence_proxy_async_smem();
            mbar_arrive(&aready[st]);
            return true;
        };
        auto epilogue = [&](int t) -> bool {
            const int st = t % kStages, buf = t & 1;
            if (!mbar_wait(&mmadone[st], (t / kStages) & 1, 208)) return false;
            tc_fence_after_sync();
            uint8_t* tile = stages + st * kTileBytes;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + buf * kBufCols;
            float v[kPairHeads][kD + 1];
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                tmem_ld16(ta + j * kN, v[j]);
                tmem_ld16(ta + j * kN + 16, v[j] + 16);
                tmem_ld1(ta + j * kN + kD, v[j] + kD);
            }
            tmem_wait_ld();
            tc_fence_before_sync();
            mbar_arrive(&tfree[buf]);
#pragma unroll
            for (int j = 0; j < kPairHeads; ++j) {
                const float inv = __frcp_rn(v[j][kD] + eps);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 w;
                    w.x = pack_bf16x2(v[j][8 * c + 0] * inv, v[j][8 * c + 1] * inv);
                    w.y = pack_bf16x2(v[j][8 * c + 2] * inv, v[j][8 * c + 3] * inv);
                    w.z = pack_bf16x2(v[j][8 * c + 4] * inv, v[j][8 * c + 5] * inv);
                    w.w = pack_bf16x2(v[j][8 * c + 6] * inv, v[j][8 * c + 7] * inv);
                    *reinterpret_cast<uint4*>(tile + sw128_offset(row, j * 4 + c)) = w;
                }
            }
            fence_proxy_async_smem();
            named_barrier_sync(1, 128);
            if (wt == 0) {
                tma_store_3d(&tmap_o, tile, pair * 64, (tile0 + t) * kTileTok, b);
                bulk_commit_group();
                bulk_wait_group_read<1>();                  // the previous tile's store has read smem
                if (t >= 1) mbar_arrive(&empty[(t - 1) % kStages]);
            }
            return true;
        };

        if (ok) ok = transform(0);
        for (int t = 0; t < nt && ok; ++t) {
            if (t + 1 < nt) ok = transform(t + 1);
            if (ok) ok = epilogue(t);
        }
        if (wt == 0) bulk_wait_group<0>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// arrives on, gives up after limit_ns, and records kErrWaitTimeout at `site`.
__global__ void wait_timeout_selftest(uint64_t limit_ns, int site)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_wait(&bar, 0, site, limit_ns);
    }
}

}  // namespace sana
