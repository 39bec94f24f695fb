// The variant fused with the QKV projection ("Sana: Efficient High-Resolution
// Image Synthesis with Linear Diffusion Transformers", section 7, on-device
// deployment: the ReLU(K)^T V reduction fused with the QKV projection), on the
// sm_100a tensor cores.  The projected Q, K and V never leave the SM: they are
// accumulated in TMEM (fp32), normalised in fp32, and only their bf16 feature
// maps reach shared memory as operands of the attention contractions.
//
//   fused_kv (F1)  CTA (s, g, b): token tiles [s*tps, (s+1)*tps) of batch b,
//                  head group g (4 heads).  Per tile of 128 tokens:
//                    [K | V] = x_tile * Wqkv[:, K and V columns of g]   (UMMA 128x256, K=2240)
//                    phi(K), V -> bf16 operands in smem
//                    S += phi(K)^T [V | 1]                              (UMMA 128x128 + 128x64)
//                  then the CTA's partial state, and the last CTA of (b, g)
//                  sums the partials in split order.
//   fused_qo (F2)  CTA (s, g, b), same tiles:
//                    Q = x_tile * Wqkv[:, Q columns of g]               (UMMA 128x128)
//                    A' = ReLU(gq * q) (bf16), r = rsqrt(mean(q^2) + eps) kept in registers
//                    D = A' [S_hi | S_lo]                               (UMMA 128x48 per head)
//                    O = r D[:, :32] / (r D[:, 32] + eps)  -> TMA store
//                  Only the B-operand build reads the states F1 wrote, so under
//                  programmatic dependent launch the Q projection overlaps F1's tail.
//
// W8A8 (template kI8): x and Wqkv arrive as int8 codes with one fp32 scale per
// token of x and per output channel of Wqkv.  The projection runs as a kind::i8
// UMMA (int32 accumulator in TMEM, exact), the epilogue dequantises
// q = acc * sx[token] * sw[channel] in fp32, and everything after that (feature
// map, state, apply: bf16 operands, fp32 accumulation) is the same as for bf16.
// A stage then covers 128 k (128 bytes of an x row, as for bf16's 64 k), a UMMA
// K = 32, and a W box is 128 k x 128 n.
//
// Operand layouts (all 128-byte swizzle, 1024-byte aligned):
//   x tile        K-major: [128 tokens][64 k] per stage (TMA 3-D map over (C, N, B))
//   W blocks      MN-major: [64 k][64 n] boxes (TMA 3-D map over (n, section, k)),
//                 consecutive boxes 8 KB apart form one N = 64 * boxes operand
//   phi(K), V     MN-major: [128 tokens][64 ch] blocks, 16 KB apart
//   A' / O        K-major:  [128 tokens][64 ch] blocks (2 heads each), 16 KB apart
#pragma once

#include "sana_common.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"

namespace sana {

namespace fz {
constexpr int kTileTok = 128;                      // UMMA M
constexpr int kGroupHeads = 4;                     // heads per CTA
constexpr int kXBytes = kTileTok * 128;            // x box: 128 tokens x 128 bytes of k = 16 KB
constexpr int kSectionBytes = 16 * 1024;           // W rows of one stage for a group's 128 n
constexpr int kBlock = kTileTok * 128;             // 128 tokens x 64 channels = 16 KB

// Element-type dependent geometry (bf16 or int8 x and Wqkv).
template <bool kI8>
struct Geom {
    static constexpr int kKStep = kI8 ? 128 : 64;      // k per stage: 128 bytes of an x row
    static constexpr int kKSlice = kI8 ? 32 : 16;      // k per UMMA (32 bytes of a K-major row)
    static constexpr int kWAtomN = kI8 ? 128 : 64;     // n in one 128-byte W row (MN-major atom)
    static constexpr int kWBox = kKStep * 128;         // W box: kKStep k rows x 128 bytes
    static constexpr int kWBoxes = 128 / kWAtomN;      // boxes per section of a group
    static_assert(kWBoxes * kWBox == kSectionBytes, "section size");
};
}  // namespace fz

// ============================================================================ F1
namespace f1 {
constexpr int kStageBytes = fz::kXBytes + 2 * fz::kSectionBytes;   // x + K section + V section
constexpr int kStages = 3;
constexpr int kOpBytes = 2 * fz::kBlock;                   // phi(K) or V: 128 tokens x 128 ch
constexpr int kOnesBytes = 16 * 128;
constexpr int kAccCols = 256;                              // [K | V] accumulator
constexpr int kKvCol = 256;                                // state accumulator at column 256
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 8;                               // two per TMEM lane quadrant
constexpr int kThreads = 32 * (2 + kEpiWarps);             // TMA, UMMA, epilogue
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 2 * kOpBytes + kOnesBytes + 1024 + 2048;
}  // namespace f1

struct F1Args {
    const float* sx;     // W8A8: per-token scales of x [B * N]
    const float* sw;     // W8A8: per-channel scales of Wqkv [3C]
    const float* gk;     // [C] or nullptr (norm off)
    float* part;         // [B][H][S][D][D+1]
    float* kv;           // [B][H][D][D+1]
    int* counters;       // [B * G], zero on entry
    int N, H, C, S, tps; // tokens per batch, heads, channels, splits, tiles per split
    float eps;
    int norm;
};

template <bool kI8>
__global__ void __launch_bounds__(f1::kThreads, 1)
fused_kv(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
         const F1Args a)
{
    using namespace f1;
    using G = fz::Geom<kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* opk = stages + kStages * kStageBytes;          // phi(K): A operand of the state MMA
    uint8_t* opv = opk + kOpBytes;                          // V: B operand
    uint8_t* ones = opv + kOpBytes;
    float* sg = (float*)(ones + kOnesBytes);                // 128 gains of the group
    float* ssw = sg + 128;                                  // W8A8: 256 K, V channel scales
    uint64_t* full = (uint64_t*)(ssw + 256);
    uint64_t* empty = full + kStages;
    uint64_t* accfull = empty + kStages;
    uint64_t* accempty = accfull + 1;
    uint64_t* opready = accempty + 1;
    uint64_t* opfree = opready + 1;
    uint64_t* kvdone = opfree + 1;
    uint32_t* tmem_slot = (uint32_t*)(kvdone + 1);
    int* last_flag = (int*)(tmem_slot + 1);

    pdl_launch_dependents();

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (a.N + fz::kTileTok - 1) / fz::kTileTok;
    const int t0 = s * a.tps;
    const int nt = min(a.tps, tiles - t0);
    const int ksteps = (a.C + G::kKStep - 1) / G::kKStep;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, 32 * kEpiWarps);
        mbar_init(opready, 32 * kEpiWarps);
        mbar_init(opfree, 1);
        mbar_init(kvdone, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
    }
    for (int i = threadIdx.x; i < kOnesBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(ones)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
        const int h = g * fz::kGroupHeads + i / kD;
        sg[i] = (a.norm && h < a.H) ? a.gk[(size_t)h * kD + (i % kD)] : 1.f;
        if (kI8) {
            const bool live = h < a.H;
            ssw[i] = live ? a.sw[a.C + g * 128 + i] : 0.f;             // K section
            ssw[128 + i] = live ? a.sw[2 * a.C + g * 128 + i] : 0.f;   // V section
        }
    }
    __syncthreads();
    if (threadIdx.x < 16)
        *reinterpret_cast<uint16_t*>(ones + sw128_offset(threadIdx.x, 0)) = 0x3F80;   // bf16 1.0
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = nt > 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && ok) {
            int64_t step = 0, last = -1;
            for (int ti = 0; ti < nt && ok; ++ti) {
                const int y = (t0 + ti) * fz::kTileTok;
                for (int kk = 0; kk < ksteps; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    if (step >= kStages)
                        ok = mbar_wait(&empty[st], (uint32_t)((step / kStages) - 1) & 1, 501);
                    if (!ok) break;
                    uint8_t* sb = stages + st * kStageBytes;
                    mbar_arrive_expect_tx(&full[st], kStageBytes);
                    tma_load_3d(sb, &tmap_x, &full[st], kk * G::kKStep, y, b);
                    const int n0 = g * 128;
#pragma unroll
                    for (int sec = 1; sec <= 2; ++sec)          // K, then V columns of the group
#pragma unroll
                        for (int j = 0; j < G::kWBoxes; ++j)
                            tma_load_3d(sb + fz::kXBytes + (sec - 1) * fz::kSectionBytes + j * G::kWBox,
                                        &tmap_w, &full[st], n0 + j * G::kWAtomN, sec,
                                        kk * G::kKStep);
                    last = step;
                }
            }
            if (!ok) {
                for (int st = 0; st < kStages; ++st) {
                    const int64_t li = last - ((last - st) % kStages + kStages) % kStages;
                    if (last >= 0 && li >= 0)
                        mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 502);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        if (lane == 0 && ok) {
            const uint32_t idesc_g = kI8 ? make_idesc_s8(128, 256, false, true)       // x K-major,
                                         : make_idesc_bf16(128, 256, false, true);  // W MN-major
            const uint32_t idesc_v = make_idesc_bf16(128, 128, true, true);    // phi(K), V MN-major
            const uint32_t idesc_1 = make_idesc_bf16(128, 64, true, true);
            const uint64_t ones_desc = make_smem_desc(smem_u32(ones), fz::kBlock, 1024, kSwizzle128B);
            int64_t step = 0;
            for (int ti = 0; ti < nt && ok; ++ti) {
                if (ti > 0) ok = mbar_wait(accempty, (uint32_t)(ti - 1) & 1, 503);
                if (!ok) break;
                tc_fence_after_sync();
                for (int kk = 0; kk < ksteps && ok; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    ok = mbar_wait(&full[st], (uint32_t)(step / kStages) & 1, 504);
                    if (!ok) break;
                    tc_fence_after_sync();
                    const uint32_t xb = smem_u32(stages + st * kStageBytes);
                    const uint32_t wb = xb + fz::kXBytes;
#pragma unroll
                    for (int k4 = 0; k4 < G::kKStep / G::kKSlice; ++k4) {
                        const uint64_t ad = make_smem_desc(xb + k4 * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_smem_desc(wb + k4 * G::kKSlice * 128, G::kWBox, 1024,
                                                           kSwizzle128B);
                        if (kI8) umma_s8(tmem, ad, bd, idesc_g, kk > 0 || k4 > 0);
                        else umma_bf16(tmem, ad, bd, idesc_g, kk > 0 || k4 > 0);
                    }
                    umma_commit(&empty[st]);
                }
                if (!ok) break;
                umma_commit(accfull);
                // the state contraction of this tile, once the epilogue has written its operands
                ok = mbar_wait(opready, (uint32_t)ti & 1, 505);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t kb = smem_u32(opk), vb = smem_u32(opv);
#pragma unroll
                for (int k4 = 0; k4 < fz::kTileTok / 16; ++k4) {
                    const uint64_t ad = make_smem_desc(kb + k4 * 2048, fz::kBlock, 1024, kSwizzle128B);
                    const uint64_t bd = make_smem_desc(vb + k4 * 2048, fz::kBlock, 1024, kSwizzle128B);
                    const bool acc = ti > 0 || k4 > 0;
                    umma_bf16(tmem + kKvCol, ad, bd, idesc_v, acc);
                    umma_bf16(tmem + kKvCol + 128, ad, ones_desc, idesc_1, acc);
                }
                umma_commit(opfree);
            }
            umma_commit(kvdone);
            mbar_wait(kvdone, 0, 506);
        }
    } else {
        // ------------------------------------------------ epilogue: phi(K), V, then the state
        // Two warps per TMEM lane quadrant: warp half 0 takes heads 0, 1 of the
        // group, half 1 heads 2, 3.
        const int et = threadIdx.x - 64;                  // 0..255
        const int half = et >> 7;
        const int q = warp & 3;                           // TMEM lane quadrant
        const int row = 32 * q + lane;                    // token row of the tile
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        for (int ti = 0; ti < nt && ok; ++ti) {
            ok = mbar_wait(accfull, (uint32_t)ti & 1, 507);
            if (ok && ti > 0) ok = mbar_wait(opfree, (uint32_t)(ti - 1) & 1, 508);
            if (!ok) break;
            tc_fence_after_sync();
            const bool row_live = (t0 + ti) * fz::kTileTok + row < a.N;
            const float sxr = (kI8 && row_live)
                ? a.sx[(int64_t)b * a.N + (t0 + ti) * fz::kTileTok + row] : 0.f;
#pragma unroll 1
            for (int j = 2 * half; j < 2 * half + 2; ++j) {
                float kx[32], vx[32];
                tmem_ld16(lane_base + 32 * j, kx);
                tmem_ld16(lane_base + 32 * j + 16, kx + 16);
                tmem_ld16(lane_base + 128 + 32 * j, vx);
                tmem_ld16(lane_base + 128 + 32 * j + 16, vx + 16);
                tmem_wait_ld();
                if (kI8) {                    // int32 accumulators -> dequantised fp32
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        kx[i] = __int2float_rn(__float_as_int(kx[i])) * sxr * ssw[j * kD + i];
                        vx[i] = __int2float_rn(__float_as_int(vx[i])) * sxr * ssw[128 + j * kD + i];
                    }
                }
                const bool live = row_live && (g * fz::kGroupHeads + j < a.H);
                if (a.norm) {
                    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        s0 = fmaf(kx[i], kx[i], s0);
                        s1 = fmaf(kx[i + 1], kx[i + 1], s1);
                        s2 = fmaf(kx[i + 2], kx[i + 2], s2);
                        s3 = fmaf(kx[i + 3], kx[i + 3], s3);
                    }
                    const float r = rsqrtf(((s0 + s1) + (s2 + s3)) * (1.f / kD) + a.eps);
#pragma unroll
                    for (int i = 0; i < 32; ++i) kx[i] = fmaxf(sg[j * kD + i] * (kx[i] * r), 0.f);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) kx[i] = fmaxf(kx[i], 0.f);
                }
                uint8_t* kblk = opk + (j >> 1) * fz::kBlock;
                uint8_t* vblk = opv + (j >> 1) * fz::kBlock;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 wk, wv;
                    if (live) {
                        wk.x = pack_bf16x2(kx[8 * c + 0], kx[8 * c + 1]);
                        wk.y = pack_bf16x2(kx[8 * c + 2], kx[8 * c + 3]);
                        wk.z = pack_bf16x2(kx[8 * c + 4], kx[8 * c + 5]);
                        wk.w = pack_bf16x2(kx[8 * c + 6], kx[8 * c + 7]);
                        wv.x = pack_bf16x2(vx[8 * c + 0], vx[8 * c + 1]);
                        wv.y = pack_bf16x2(vx[8 * c + 2], vx[8 * c + 3]);
                        wv.z = pack_bf16x2(vx[8 * c + 4], vx[8 * c + 5]);
                        wv.w = pack_bf16x2(vx[8 * c + 6], vx[8 * c + 7]);
                    } else {
                        wk = make_uint4(0, 0, 0, 0);
                        wv = make_uint4(0, 0, 0, 0);
                    }
                    const uint32_t off = sw128_offset(row, (j & 1) * 4 + c);
                    *reinterpret_cast<uint4*>(kblk + off) = wk;
                    *reinterpret_cast<uint4*>(vblk + off) = wv;
                }
            }
            tc_fence_before_sync();
            mbar_arrive(accempty);
            fence_proxy_async_smem();
            mbar_arrive(opready);
        }
        if (ok) ok = mbar_wait(kvdone, 0, 509);
        // Each thread decided `ok` on its own waits; the half-0 threads agree on it
        // before the named barriers below, so none of them waits at one alone.
        if (half == 0) ok = named_barrier_and(1, 128, ok);
        if (ok && half == 0) {
            // the CTA's partial state: diagonal blocks of the state accumulator
            tc_fence_after_sync();
            const int h = g * fz::kGroupHeads + q;
            float v[32], ks;
            tmem_ld16(lane_base + kKvCol + 32 * q, v);
            tmem_ld16(lane_base + kKvCol + 32 * q + 16, v + 16);
            tmem_ld1(lane_base + kKvCol + 128, &ks);
            tmem_wait_ld();
            if (h < a.H) {
                float* o = a.part + (((size_t)b * a.H + h) * a.S + s) * kStateFloats + lane * kDP;
#pragma unroll
                for (int e = 0; e < kD; ++e) o[e] = v[e];
                o[kD] = ks;
            }
            __threadfence();
            named_barrier_sync(1, 128);
            const int row_id = b * gridDim.y + g;
            const int nsplits = (tiles + a.tps - 1) / a.tps;
            if (et == 0) *last_flag = (atomicAdd(&a.counters[row_id], 1) == nsplits - 1);
            named_barrier_sync(1, 128);
            if (*last_flag) {
                __threadfence();
                for (int idx = et; idx < fz::kGroupHeads * (kStateFloats / 4); idx += 128) {
                    const int hh = g * fz::kGroupHeads + idx / (kStateFloats / 4);
                    const int e4 = idx % (kStateFloats / 4);
                    if (hh >= a.H) continue;
                    const float4* pp = reinterpret_cast<const float4*>(
                        a.part + ((size_t)b * a.H + hh) * a.S * kStateFloats) + e4;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int sp = 0; sp < nsplits; ++sp) {
                        const float4 x = __ldcg(pp + (size_t)sp * (kStateFloats / 4));
                        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
                    }
                    reinterpret_cast<float4*>(a.kv + ((size_t)b * a.H + hh) * kStateFloats)[e4] = acc;
                }
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

// ============================================================================ F2
namespace f2 {
constexpr int kStageBytes = fz::kXBytes + fz::kSectionBytes;   // x + Q section
constexpr int kStages = 5;
constexpr int kN = 48;                                     // 32 value columns, normaliser, padding
constexpr int kBopBytes = kN * 128;                        // per head
constexpr int kQoBytes = 2 * fz::kBlock;                   // states, then A' / O staging
constexpr int kStateBytes = fz::kGroupHeads * kStateFloats * 4;   // staged in the qo buffer
constexpr int kAccCols = 128;                              // Q accumulator (two buffers)
constexpr int kDCol = 256;                                 // apply accumulators at column 256
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + fz::kGroupHeads * kBopBytes +
                           kQoBytes + 512 + 2048;
static_assert(kStateBytes <= kQoBytes, "states must fit the staging buffer");
}  // namespace f2

struct F2Args {
    const float* sx;     // W8A8: per-token scales of x [B * N]
    const float* sw;     // W8A8: per-channel scales of Wqkv [3C]
    const float* kv;     // states [B][H][D][D+1] (F1's output)
    const float* gq;     // [C] or nullptr
    int N, H, C, tps;
    float eps;
    int norm;
};

template <bool kI8>
__global__ void __launch_bounds__(f2::kThreads, 1)
fused_qo(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
         const __grid_constant__ CUtensorMap tmap_o, const F2Args a)
{
    using namespace f2;
    using G = fz::Geom<kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* stages = smem;
    uint8_t* bop = stages + kStages * kStageBytes;
    uint8_t* qo = bop + fz::kGroupHeads * kBopBytes;
    float* sstate = (float*)qo;                             // states before the first tile
    float* sg = (float*)(qo + kQoBytes);                    // 128 gains
    float* ssw = sg + 128;                                  // W8A8: 128 Q channel scales
    uint64_t* full = (uint64_t*)(ssw + 128);
    uint64_t* empty = full + kStages;
    uint64_t* accfull = empty + kStages;                    // [2]
    uint64_t* accempty = accfull + 2;                       // [2]
    uint64_t* opready = accempty + 2;
    uint64_t* ddone = opready + 1;
    uint64_t* bready = ddone + 1;
    uint64_t* sready = bready + 1;
    uint64_t* drain = sready + 1;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (a.N + fz::kTileTok - 1) / fz::kTileTok;
    const int t0 = s * a.tps;
    const int nt = min(a.tps, tiles - t0);
    const int ksteps = (a.C + G::kKStep - 1) / G::kKStep;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 32 * kEpiWarps);
        }
        mbar_init(opready, 32 * kEpiWarps);
        mbar_init(ddone, 1);
        mbar_init(bready, 32 * kEpiWarps);
        mbar_init(sready, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_o);
    }
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
        const int h = g * fz::kGroupHeads + i / kD;
        sg[i] = (a.norm && h < a.H) ? a.gq[(size_t)h * kD + (i % kD)] : 1.f;
        if (kI8) ssw[i] = h < a.H ? a.sw[g * 128 + i] : 0.f;       // Q section
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
            int64_t step = 0, last = -1;
            for (int ti = 0; ti < nt && ok; ++ti) {
                const int y = (t0 + ti) * fz::kTileTok;
                for (int kk = 0; kk < ksteps; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    if (step >= kStages)
                        ok = mbar_wait(&empty[st], (uint32_t)((step / kStages) - 1) & 1, 601);
                    if (!ok) break;
                    uint8_t* sb = stages + st * kStageBytes;
                    mbar_arrive_expect_tx(&full[st], kStageBytes);
                    tma_load_3d(sb, &tmap_x, &full[st], kk * G::kKStep, y, b);
#pragma unroll
                    for (int j = 0; j < G::kWBoxes; ++j)        // Q columns of the group
                        tma_load_3d(sb + fz::kXBytes + j * G::kWBox, &tmap_w, &full[st],
                                    g * 128 + j * G::kWAtomN, 0, kk * G::kKStep);
                    last = step;
                }
            }
            if (!ok) {
                for (int st = 0; st < kStages; ++st) {
                    const int64_t li = last - ((last - st) % kStages + kStages) % kStages;
                    if (last >= 0 && li >= 0)
                        mbar_wait(&full[st], (uint32_t)(li / kStages) & 1, 602);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ UMMA issuer
        // Order: GEMM(0), GEMM(1), apply(0), GEMM(2), apply(1), ...  The apply of a
        // tile is issued after the next tile's projection, so the tensor pipe keeps
        // busy while the epilogue turns the tile's Q into the A' operand.
        if (lane == 0 && ok) {
            const uint32_t idesc_g = kI8 ? make_idesc_s8(128, 128, false, true)
                                         : make_idesc_bf16(128, 128, false, true);
            const uint32_t idesc_a = make_idesc_bf16(128, kN, false, false);
            int64_t step = 0;
            auto gemm = [&](int ti) -> bool {
                const int ab = ti & 1;
                if (ti >= 2 && !mbar_wait(&accempty[ab], (uint32_t)((ti >> 1) - 1) & 1, 603))
                    return false;
                tc_fence_after_sync();
                for (int kk = 0; kk < ksteps; ++kk, ++step) {
                    const int st = (int)(step % kStages);
                    if (!mbar_wait(&full[st], (uint32_t)(step / kStages) & 1, 604)) return false;
                    tc_fence_after_sync();
                    const uint32_t xb = smem_u32(stages + st * kStageBytes);
                    const uint32_t wb = xb + fz::kXBytes;
#pragma unroll
                    for (int k4 = 0; k4 < G::kKStep / G::kKSlice; ++k4) {
                        const uint64_t ad = make_smem_desc(xb + k4 * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_smem_desc(wb + k4 * G::kKSlice * 128, G::kWBox, 1024,
                                                           kSwizzle128B);
                        if (kI8) umma_s8(tmem + ab * kAccCols, ad, bd, idesc_g, kk > 0 || k4 > 0);
                        else umma_bf16(tmem + ab * kAccCols, ad, bd, idesc_g, kk > 0 || k4 > 0);
                    }
                    umma_commit(&empty[st]);
                }
                umma_commit(&accfull[ab]);
                return true;
            };
            auto apply = [&](int ti) -> bool {
                if (ti == 0 && !mbar_wait(bready, 0, 605)) return false;
                if (!mbar_wait(opready, (uint32_t)ti & 1, 606)) return false;
                tc_fence_after_sync();
                const uint32_t qb = smem_u32(qo), bb0 = smem_u32(bop);
#pragma unroll
                for (int j = 0; j < fz::kGroupHeads; ++j) {
                    const uint32_t d = tmem + kDCol + j * kN;
                    const uint32_t ab = qb + (j >> 1) * fz::kBlock + (j & 1) * 64;
                    const uint32_t bb = bb0 + j * kBopBytes;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t ad = make_smem_desc(ab + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t hi = make_smem_desc(bb + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t lo = make_smem_desc(bb + 64 + kk * 32, 16, 1024, kSwizzle128B);
                        umma_bf16(d, ad, hi, idesc_a, kk > 0);
                        umma_bf16(d, ad, lo, idesc_a, true);
                    }
                }
                umma_commit(ddone);
                return true;
            };
            for (int ti = 0; ti <= nt && ok; ++ti) {
                if (ti < nt) ok = gemm(ti);
                if (ok && ti >= 1) ok = apply(ti - 1);
            }
            umma_commit(drain);
            mbar_wait(drain, 0, 607);
        }
    } else {
        // ------------------------------------------------ epilogue (two warps per quadrant:
        // half 0 takes heads 0, 1 of the group, half 1 heads 2, 3)
        const int et = threadIdx.x - 64;                  // 0..255
        const int half = et >> 7;
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        // B operand of the apply contraction from the group's fp32 states (F1's output)
        pdl_wait_primary();
        const int nh = min(fz::kGroupHeads, a.H - g * fz::kGroupHeads);
        if (et == 0) {
            const uint32_t bytes = (uint32_t)(nh * kStateFloats * 4);
            mbar_arrive_expect_tx(sready, bytes);
            bulk_load(sstate, a.kv + ((size_t)b * a.H + g * fz::kGroupHeads) * kStateFloats, bytes,
                      sready);
        }
        ok = ok && mbar_wait(sready, 0, 608);
        for (int idx = et; idx < fz::kGroupHeads * kN * 8; idx += 32 * kEpiWarps) {
            const int j = idx / (kN * 8), rem = idx % (kN * 8), n = rem >> 3, ch = rem & 7;
            const float* src = sstate + j * kStateFloats;
            float vals[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int dd = (ch & 3) * 8 + u;
                const float x = (ok && j < nh && n <= kD) ? src[dd * kDP + n] : 0.f;
                const float hi = __bfloat162float(__float2bfloat16_rn(x));
                vals[u] = (ch < 4) ? hi : (x - hi);
            }
            uint4 w;
            w.x = pack_bf16x2(vals[0], vals[1]);
            w.y = pack_bf16x2(vals[2], vals[3]);
            w.z = pack_bf16x2(vals[4], vals[5]);
            w.w = pack_bf16x2(vals[6], vals[7]);
            *reinterpret_cast<uint4*>(bop + j * kBopBytes + sw128_offset(n, ch)) = w;
        }
        fence_proxy_async_smem();
        // The states in qo have been read.  Every epilogue thread reaches each named
        // barrier from here on, and the barriers also settle `ok` (each thread's
        // waits are bounded on their own), so the threads leave the loop together.
        ok = named_barrier_and(1, 32 * kEpiWarps, ok);
        mbar_arrive(bready);

        for (int ti = 0; ti < nt && ok; ++ti) {
            const int ab = ti & 1;
            bool wok = mbar_wait(&accfull[ab], (uint32_t)(ti >> 1) & 1, 609);
            // the previous tile's O store must have read the staging buffer
            if (et == 0) bulk_wait_group_read<0>();
            ok = named_barrier_and(1, 32 * kEpiWarps, wok);
            if (!ok) break;
            tc_fence_after_sync();
            const bool row_live = (t0 + ti) * fz::kTileTok + row < a.N;
            const float sxr = (kI8 && row_live)
                ? a.sx[(int64_t)b * a.N + (t0 + ti) * fz::kTileTok + row] : 0.f;
            float rq[2];
#pragma unroll 1
            for (int j = 2 * half; j < 2 * half + 2; ++j) {
                float x[32];
                tmem_ld16(lane_base + ab * kAccCols + 32 * j, x);
                tmem_ld16(lane_base + ab * kAccCols + 32 * j + 16, x + 16);
                tmem_wait_ld();
                if (kI8) {                    // int32 accumulators -> dequantised fp32
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        x[i] = __int2float_rn(__float_as_int(x[i])) * sxr * ssw[j * kD + i];
                }
                const bool live = row_live && (g * fz::kGroupHeads + j < a.H);
                float r = 1.f;
                if (a.norm) {
                    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        s0 = fmaf(x[i], x[i], s0);
                        s1 = fmaf(x[i + 1], x[i + 1], s1);
                        s2 = fmaf(x[i + 2], x[i + 2], s2);
                        s3 = fmaf(x[i + 3], x[i + 3], s3);
                    }
                    r = rsqrtf(((s0 + s1) + (s2 + s3)) * (1.f / kD) + a.eps);
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = fmaxf(sg[j * kD + i] * x[i], 0.f);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = fmaxf(x[i], 0.f);
                }
                rq[j & 1] = r;
                uint8_t* blk = qo + (j >> 1) * fz::kBlock;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (live) {
                        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
                        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
                        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
                        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
                    }
                    *reinterpret_cast<uint4*>(blk + sw128_offset(row, (j & 1) * 4 + c)) = w;
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&accempty[ab]);
            fence_proxy_async_smem();
            mbar_arrive(opready);
            // O = r D[:, :32] / (r D[:, 32] + eps), written over the A' operand
            wok = mbar_wait(ddone, (uint32_t)ti & 1, 610);
            tc_fence_after_sync();
#pragma unroll 1
            for (int j = 2 * half; j < 2 * half + 2 && wok; ++j) {
                float v[kD + 1];
                tmem_ld16(lane_base + kDCol + j * kN, v);
                tmem_ld16(lane_base + kDCol + j * kN + 16, v + 16);
                tmem_ld1(lane_base + kDCol + j * kN + kD, v + kD);
                tmem_wait_ld();
                const float scale = rq[j & 1] * __frcp_rn(fmaf(rq[j & 1], v[kD], a.eps));
                uint8_t* blk = qo + (j >> 1) * fz::kBlock;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * c + 0] * scale, v[8 * c + 1] * scale);
                    w.y = pack_bf16x2(v[8 * c + 2] * scale, v[8 * c + 3] * scale);
                    w.z = pack_bf16x2(v[8 * c + 4] * scale, v[8 * c + 5] * scale);
                    w.w = pack_bf16x2(v[8 * c + 6] * scale, v[8 * c + 7] * scale);
                    *reinterpret_cast<uint4*>(blk + sw128_offset(row, (j & 1) * 4 + c)) = w;
                }
            }
            tc_fence_before_sync();
            fence_proxy_async_smem();
            ok = named_barrier_and(1, 32 * kEpiWarps, wok);
            if (ok && et == 0) {
                const int y = (t0 + ti) * fz::kTileTok;
                tma_store_3d(&tmap_o, qo, g * 128, y, b);
                if (g * 128 + 64 < a.C)                       // no store that starts past C
                    tma_store_3d(&tmap_o, qo + fz::kBlock, g * 128 + 64, y, b);
                bulk_commit_group();
            }
        }
        if (et == 0) bulk_wait_group<0>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sana
