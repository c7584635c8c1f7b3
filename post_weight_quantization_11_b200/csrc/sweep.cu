// Layer quantization driver and the intra-block column sweep -- "INT4/INT8
// 量化推理" sec. 三 (quantize column by column, push the error onto the
// not-yet-quantized columns), "GPTQ / AWQ / SqueezeLLM" sec. 一 (process in
// blocks), "大模型量化的“校准”艺术" sec. 2.2 steps 1-5.
//
// Per 128-column block b (columns j0 .. j0+127, sweep order):
//   block_sweep:  every row runs the 128 sequential steps with the block's
//                 columns in registers (8 lanes per row, 16 columns per lane)
//                 and U's 128x128 diagonal block in shared memory; writes the
//                 codes, group scales/zeros, the scaled errors E (rows x 128)
//                 and accumulates sum E_j^2 per row.
//   block_update: W[:, cols] -= E . U[rows of E, cols], deferred in two
//                 levels (see gptq_quantize_layer below)
// Rows are independent given U, so a block's sweep is parallel over rows and
// only the chain of blocks is sequential.
#include "common.cuh"
#include "quant_common.cuh"
#include "tc_common.cuh"
#include "update.cuh"

namespace gptq {

constexpr int SW_B = 128;          // block width (columns)
constexpr int SW_LPR = 8;          // lanes per row
constexpr int SW_CPL = SW_B / SW_LPR;   // columns per lane (16)
constexpr int SW_Q4 = SW_CPL / 4;       // float4 chunks per lane (4)
constexpr int SW_THREADS = 128;
constexpr int SW_RPL = 2;          // rows per lane group
constexpr int SW_ROWS = SW_RPL * SW_THREADS / SW_LPR;   // rows per CTA
constexpr unsigned FULL = 0xffffffffu;

// W_work[r][k] = float(W[r][perm[k]])
template <typename T>
__global__ void init_work_kernel(const T* __restrict__ W, const int32_t* __restrict__ perm,
                                 int64_t m, int64_t d, float* __restrict__ Wk)
{
    const int64_t total = m * d;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = i / d, k = i - r * d;
        const int64_t src = perm ? int64_t(perm[k]) : k;
        const bool in = src >= 0 && src < d;          // a bad index is not followed
        if (!in) atomicCAS(&g_device_status, 0, kErrIndex);
        Wk[i] = in ? float(W[r * d + src]) : 0.f;
    }
}

// One 128-column block of the sweep for all rows.  8 lanes per row, each lane
// holding 16 consecutive columns of SW_RPL rows in registers (rows g, g+4 ..
// of its warp's rows).  One row per lane group: 16 rows per CTA, so a layer
// of a few thousand rows puts two CTAs (eight independent decision chains per
// scheduler pair) on most SMs, and the chains of different warps hide each
// other's latency.  U's 128x128
// diagonal block (its strictly-lower part zeroed) and 1/U_jj live in shared
// memory.  Step j: every lane of a row takes the same fp32 decision on column
// j (quant_code_fast: no division) and applies w[k] -= E_j U[j][k] to its
// columns; the next column's value is shuffled from its owner before the
// decision and each lane applies the one correction itself, so the shuffle
// is off the dependency chain.  At a group's first column the group's
// min/max is reduced over the row's lanes (lanes outside the group
// contribute 0, neutral since the range includes 0).  The outer loop over the
// 8 owner lanes is not unrolled, which keeps the kernel's code small.
// STATIC: the group parameters were set before the sweep (static groups, or
// one group per row); the kernel loads them at each group start inside the
// block and at the block's first column instead of reducing min/max.  GS is
// then min(group size, 128) and gsz the group size.
// The 128 sequential steps of one block for this lane's rows: w holds the
// lane's 16 columns of each row (updated through every earlier column), Us
// the block's diagonal U block (strictly-lower part zeroed, chunk-major) and
// rdiag 1/U_jj.  Writes the group scales/zeros of groups starting in the
// block (dynamic groups) and leaves in Ev/cp the errors and codes of the
// 16 columns this lane owns, in loss the row's sum of E_j^2 over the block.
template <int GS, bool STATIC>
__device__ __forceinline__ void sweep_core(const float* __restrict__ Us,
                                           const float* __restrict__ rdiag,
                                           float (&w)[SW_RPL][SW_CPL],
                                           const int64_t (&row)[SW_RPL],
                                           const bool (&valid)[SW_RPL], int sub, int src_base,
                                           int64_t G, int64_t gsz, int64_t j0, float maxqf,
                                           __half* __restrict__ scales,
                                           uint8_t* __restrict__ zeros,
                                           float (&Ev)[SW_RPL][SW_CPL],
                                           uint32_t (&cp)[SW_RPL][SW_Q4], float (&loss)[SW_RPL])
{
    GroupQ gq[SW_RPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) {
#pragma unroll
        for (int q = 0; q < SW_Q4; ++q) cp[r][q] = 0u;
        loss[r] = 0.f;
        gq[r].s = 1.f; gq[r].z = 0.f; gq[r].r = 1.f; gq[r].h = __float2half(1.f);
    }
    float xn[SW_RPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) xn[r] = __shfl_sync(FULL, w[r][0], src_base);

#pragma unroll 1
    for (int jo = 0; jo < SW_LPR; ++jo) {
#pragma unroll
        for (int ji = 0; ji < SW_CPL; ++ji) {
            const int j = jo * SW_CPL + ji;
            if (STATIC && ji == 0 && (jo * SW_CPL) % GS == 0) {
                const int64_t gi = (j0 + j) / gsz;
#pragma unroll
                for (int r = 0; r < SW_RPL; ++r) {
                    if (valid[r]) {
                        const __half h = scales[row[r] * G + gi];
                        gq[r].h = h;
                        gq[r].s = __half2float(h);
                        gq[r].z = float(zeros[row[r] * G + gi]);
                        gq[r].r = __frcp_rn(gq[r].s);
                    }
                }
            } else if (ji == 0 && (jo * SW_CPL) % GS == 0) {
                constexpr int span = GS / SW_CPL;            // lanes covering one group
                const bool in_group = sub >= jo && sub < jo + span;
#pragma unroll
                for (int r = 0; r < SW_RPL; ++r) {
                    float mn = 0.f, mx = 0.f;
                    if (in_group) {
#pragma unroll
                        for (int q = 0; q < SW_CPL; ++q) { mn = fminf(mn, w[r][q]); mx = fmaxf(mx, w[r][q]); }
                    }
#pragma unroll
                    for (int o = 1; o < SW_LPR; o <<= 1) {
                        mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
                        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
                    }
                    gq[r] = group_params(mn, mx, maxqf);
                    if (valid[r] && sub == jo) {
                        const int64_t gi = (j0 + j) / GS;
                        scales[row[r] * G + gi] = gq[r].h;
                        zeros[row[r] * G + gi] = (uint8_t)gq[r].z;
                    }
                }
            }
            // next column's values before this column's correction (off the chain)
            float xpre[SW_RPL];
#pragma unroll
            for (int r = 0; r < SW_RPL; ++r) xpre[r] = 0.f;
            float unext = 0.f;
#pragma unroll
            for (int r = 0; r < SW_RPL; ++r) {
                if (ji + 1 < SW_CPL) xpre[r] = __shfl_sync(FULL, w[r][ji + 1], src_base | jo);
                else if (jo + 1 < SW_LPR) xpre[r] = __shfl_sync(FULL, w[r][0], src_base | (jo + 1));
            }
            if (j + 1 < SW_B) {
                const int f = (j + 1) >> 2;
                unext = Us[j * SW_B + ((f % SW_Q4) * SW_LPR + f / SW_Q4) * 4 + ((j + 1) & 3)];
            }
            const float rdj = rdiag[j];
            float Ej[SW_RPL];
#pragma unroll
            for (int r = 0; r < SW_RPL; ++r) {
                const float x = xn[r];
                const float c = quant_code_fast(x, gq[r], maxqf);
                const float q = gq[r].s * (c - gq[r].z);
                Ej[r] = (x - q) * rdj;
                loss[r] = fmaf(Ej[r], Ej[r], loss[r]);
                if (sub == jo) {
                    Ev[r][ji] = Ej[r];
                    cp[r][ji / 4] |= code_byte(c) << (8 * (ji % 4));
                }
                xn[r] = fmaf(-Ej[r], unext, xpre[r]);
            }
            const float4* urow = reinterpret_cast<const float4*>(Us + j * SW_B);
#pragma unroll
            for (int q4 = 0; q4 < SW_Q4; ++q4) {
                const float4 u = urow[q4 * SW_LPR + sub];
#pragma unroll
                for (int r = 0; r < SW_RPL; ++r) {
                    w[r][4 * q4 + 0] = fmaf(-Ej[r], u.x, w[r][4 * q4 + 0]);
                    w[r][4 * q4 + 1] = fmaf(-Ej[r], u.y, w[r][4 * q4 + 1]);
                    w[r][4 * q4 + 2] = fmaf(-Ej[r], u.z, w[r][4 * q4 + 2]);
                    w[r][4 * q4 + 3] = fmaf(-Ej[r], u.w, w[r][4 * q4 + 3]);
                }
            }
        }
    }
}

template <int GS, bool STATIC>
__global__ void __launch_bounds__(SW_THREADS)
block_sweep_kernel(const float* __restrict__ Wk, const float* __restrict__ U, int64_t m, int64_t d,
                   int64_t gsz, int64_t j0, float maxqf, uint8_t* __restrict__ codes,
                   __half* __restrict__ scales, uint8_t* __restrict__ zeros,
                   float* __restrict__ Eh_out, float* __restrict__ El_out, int64_t ldE,
                   float* __restrict__ row_loss, int first_block)
{
    extern __shared__ __align__(16) float smem[];
    float* Us = smem;                        // 128 x 128, strictly-lower part zeroed, swizzled
    float* rdiag = smem + SW_B * SW_B;       // 128: 1 / U_jj
    const int tid = threadIdx.x;
    // Row j of the block is stored chunk-major: float4 chunk q of lane `sub`'s
    // 16 columns at position q*8 + sub, so the 8 lanes of a row read 128
    // contiguous bytes per float4 load.  All loads of a half block first, then
    // the stores.
    constexpr int UPT = SW_B * SW_B / 4 / SW_THREADS / 2;   // float4 per thread per half
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
        float4 uv[UPT];
#pragma unroll
        for (int i = 0; i < UPT; ++i) {
            const int idx = (tid + (hb * UPT + i) * SW_THREADS) * 4;
            uv[i] = *reinterpret_cast<const float4*>(U + (j0 + idx / SW_B) * d + j0 + idx % SW_B);
        }
#pragma unroll
        for (int i = 0; i < UPT; ++i) {
            const int idx = (tid + (hb * UPT + i) * SW_THREADS) * 4;
            const int a = idx / SW_B, b = idx % SW_B;
            float4 v = uv[i];
            if (b + 0 < a) v.x = 0.f;
            if (b + 1 < a) v.y = 0.f;
            if (b + 2 < a) v.z = 0.f;
            if (b + 3 < a) v.w = 0.f;
            const int f = b / 4;                 // natural float4 index in the row
            *reinterpret_cast<float4*>(Us + a * SW_B + ((f % SW_Q4) * SW_LPR + f / SW_Q4) * 4) = v;
        }
    }
    if (tid < SW_B) rdiag[tid] = 1.0f / U[(j0 + tid) * d + j0 + tid];

    const int lane = tid & 31, sub = lane & (SW_LPR - 1);
    const int src_base = lane & ~(SW_LPR - 1);
    const int64_t rbase = int64_t(blockIdx.x) * SW_ROWS + (tid >> 5) * (32 / SW_LPR * SW_RPL) +
                          lane / SW_LPR;
    int64_t row[SW_RPL];
    bool valid[SW_RPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) { row[r] = rbase + (32 / SW_LPR) * r; valid[r] = row[r] < m; }
    const int64_t G = d / gsz;

    float w[SW_RPL][SW_CPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) {
        if (valid[r]) {
            const float4* p = reinterpret_cast<const float4*>(Wk + row[r] * d + j0 + SW_CPL * sub);
#pragma unroll
            for (int q = 0; q < SW_Q4; ++q) {
                const float4 v = p[q];
                w[r][4 * q] = v.x; w[r][4 * q + 1] = v.y; w[r][4 * q + 2] = v.z; w[r][4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < SW_CPL; ++q) w[r][q] = 0.f;
        }
    }
    __syncthreads();

    float Ev[SW_RPL][SW_CPL];
    uint32_t cp[SW_RPL][SW_Q4];
    float loss[SW_RPL];
    sweep_core<GS, STATIC>(Us, rdiag, w, row, valid, sub, src_base, G, gsz, j0, maxqf, scales,
                           zeros, Ev, cp, loss);
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) {
        if (!valid[r]) continue;
        static_assert(SW_CPL % 16 == 0, "codes of a lane are stored as whole uint4");
#pragma unroll
        for (int u = 0; u < SW_CPL / 16; ++u)
            *reinterpret_cast<uint4*>(codes + row[r] * d + j0 + SW_CPL * sub + 16 * u) =
                make_uint4(cp[r][4 * u], cp[r][4 * u + 1], cp[r][4 * u + 2], cp[r][4 * u + 3]);
        // E split into its TF32 head and fp32 remainder for the tensor-core update
        float4* hdst = reinterpret_cast<float4*>(Eh_out + row[r] * ldE + SW_CPL * sub);
        float4* ldst = reinterpret_cast<float4*>(El_out + row[r] * ldE + SW_CPL * sub);
#pragma unroll
        for (int q = 0; q < SW_Q4; ++q) {
            float4 h, l;
            h.x = tf32_round(Ev[r][4 * q + 0]); l.x = Ev[r][4 * q + 0] - h.x;
            h.y = tf32_round(Ev[r][4 * q + 1]); l.y = Ev[r][4 * q + 1] - h.y;
            h.z = tf32_round(Ev[r][4 * q + 2]); l.z = Ev[r][4 * q + 2] - h.z;
            h.w = tf32_round(Ev[r][4 * q + 3]); l.w = Ev[r][4 * q + 3] - h.w;
            hdst[q] = h;
            ldst[q] = l;
        }
        if (row_loss && sub == 0)
            row_loss[row[r]] = first_block ? loss[r] : row_loss[row[r]] + loss[r];
    }
}

// One 512-column outer block of the sweep, fused: a CTA keeps its 32 rows of
// the outer block in shared memory and sweeps its 128-column blocks in turn
// (sweep_core); each block's errors are applied to the CTA's rows' later
// columns of the outer block (for every block pair the correction sum
// E_b U[b rows, cols] first, then one subtraction from W).  Rows are independent given
// U, so this needs no other CTA; it replaces a sweep launch per block and a
// near-update launch per block but the last.  The errors also leave (as the
// TF32 head and fp32 remainder) for the tensor-core update of the columns
// beyond the outer block.
// Warp roles (8 warps): warps 0-3 sweep; warps 4-7 apply block b-1's errors
// to blocks b+1.. while block b is swept (phase A), then every warp applies
// block b's errors to block b+1, the next block to sweep (phase B).  A
// column receives the corrections of the earlier blocks in block order.
// U tiles come with 16-byte async copies: the diagonal tile of the next
// block during phase B, the off-diagonal tiles as 64-row halves through two
// buffers (the next half copied while one is in use; phase B's tile is
// copied at the end of phase A).  A diagonal tile is stored chunk-major
// (sweep_core's layout) and its strictly lower part is left as U holds it:
// sweep_core's corrections to columns already decided are never read.
// The updates are m16n8k8 tensor-core products (mma.sync) in split TF32:
// three products per pair of operands, fp32 accumulation, as the unfused
// tensor-core update.
//   shared memory: Ws   32 rows x (512 + 4) fp32   (the CTA's rows of the outer block)
//                  D    128 x 128 + 128 fp32       (diagonal tile, then 1/U_jj)
//                  H    2 x 64 x (128 + 8) fp32    (halves of off-diagonal tiles)
//                  Es   32 x (128 + 4) fp32        (a block's errors, row-major)
constexpr int OS_THREADS = 2 * SW_THREADS;
constexpr int OS_WLD = UPD_OUTER * SW_B + 4;
constexpr int OS_DBUF = SW_B * SW_B + SW_B;
// Row strides of a half tile (OS_HLD) and of Es (OS_ELD), so that the 32
// lanes of an m16n8k8 fragment load hit 32 different banks: lane (g, t) reads
// Es at 4 g + t and a half tile at 8 t + g (mod 32) past the fragment's base.
constexpr int OS_HLD = SW_B + 8;
constexpr int OS_ELD = SW_B + 4;
constexpr int OS_HALF = (SW_B / 2) * OS_HLD;
constexpr size_t OS_SMEM = sizeof(float) * (size_t(SW_ROWS) * OS_WLD + OS_DBUF + 2 * OS_HALF +
                                             SW_ROWS * OS_ELD);
static_assert(SW_ROWS == 32 && SW_THREADS == 128, "update tilings below assume 32 rows");

// D (16x8, fp32) += A (16x8) B (8x8) on the tensor cores, TF32 inputs (mma.sync).
__device__ __forceinline__ void mma_tf32_m16n8k8(float (&c)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x = head + tail: head its TF32 truncation, tail the exact fp32 remainder
// (whose own TF32 part the tensor core reads); the three products
// head*head + head*tail + tail*head leave out tail*tail, about 2^-20 of x y.
__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo)
{
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}

// acc (this warp's 32 rows x 8 NT columns, as 2 x NT m16n8 tiles) +=
// E[rows, k0 .. k0 + 64) . Hb[0 .. 64, c0w .. c0w + 8 NT) in split TF32:
// E row-major in Es (row stride OS_ELD), the half tile row-major in Hb
// (row stride OS_HLD).
template <int NT>
__device__ __forceinline__ void os_mma_half(float (&acc)[2][NT][4], const float* Es,
                                            const float* Hb, int k0, int c0w, int lane)
{
    const int g = lane >> 2, tg = lane & 3;
#pragma unroll 2
    for (int kk = 0; kk < SW_B / 2; kk += 8) {
        uint32_t ah[2][4], al[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const float* er = Es + (16 * mt + g) * OS_ELD + k0 + kk + tg;
            const float av[4] = {er[0], er[8 * OS_ELD], er[4], er[8 * OS_ELD + 4]};
#pragma unroll
            for (int v = 0; v < 4; ++v) tf32_split(av[v], ah[mt][v], al[mt][v]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float* br = Hb + (kk + tg) * OS_HLD + c0w + 8 * nt + g;
            uint32_t bh0, bl0, bh1, bl1;
            tf32_split(br[0], bh0, bl0);
            tf32_split(br[4 * OS_HLD], bh1, bl1);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                mma_tf32_m16n8k8(acc[mt][nt], ah[mt], bh0, bh1);
                mma_tf32_m16n8k8(acc[mt][nt], ah[mt], bl0, bl1);
                mma_tf32_m16n8k8(acc[mt][nt], al[mt], bh0, bh1);
            }
        }
    }
}

// Ws[rows, b2 block, c0w .. c0w + 8 NT) -= acc
template <int NT>
__device__ __forceinline__ void os_mma_subtract(float* Ws, int b2, const float (&acc)[2][NT][4],
                                                int c0w, int lane)
{
    const int g = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float2* p = reinterpret_cast<float2*>(Ws + (16 * mt + g + 8 * hf) * OS_WLD +
                                                      b2 * SW_B + c0w + 8 * nt + 2 * tg);
                const float2 a = *p;
                *p = make_float2(a.x - acc[mt][nt][2 * hf], a.y - acc[mt][nt][2 * hf + 1]);
            }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// every group this thread committed has landed
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// every group this thread committed but the newest has landed
__device__ __forceinline__ void cp_async_wait_all_but_newest()
{
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}
// barrier among the nthreads threads (whole warps) that use this id
__device__ __forceinline__ void bar_named(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Thread t of nthr (a multiple of 32): copies of the diagonal tile at (j0, j0)
// into D, chunk-major.  Thread t copies the 16-byte chunk (t % 32) of rows
// t / 32, t / 32 + nthr / 32, ...
__device__ __forceinline__ void os_copy_diag(const float* __restrict__ U, int64_t d, int64_t j0,
                                             float* D, int t, int nthr)
{
    const int f = t & 31;
    const int step = nthr >> 5;
    const float* src = U + (j0 + (t >> 5)) * d + j0 + 4 * f;
    float* dst = D + (t >> 5) * SW_B + ((f % SW_Q4) * SW_LPR + f / SW_Q4) * 4;
#pragma unroll 4
    for (int a = t >> 5; a < SW_B; a += step) {
        cp_async16(dst, src);
        src += step * d;
        dst += step * SW_B;
    }
}

// Thread t of nthr: copies of rows [k0, k0 + 64) x columns [c0, c0 + 128) of
// U into H, row-major (row stride OS_HLD).
__device__ __forceinline__ void os_copy_half(const float* __restrict__ U, int64_t d, int64_t k0,
                                             int64_t c0, float* H, int t, int nthr)
{
    const int f = t & 31;
    const int step = nthr >> 5;
    const float* src = U + (k0 + (t >> 5)) * d + c0 + 4 * f;
    float* dst = H + (t >> 5) * OS_HLD + 4 * f;
#pragma unroll 4
    for (int a = t >> 5; a < SW_B / 2; a += step) {
        cp_async16(dst, src);
        src += step * d;
        dst += step * OS_HLD;
    }
}

template <int GS, bool STATIC>
__global__ void __launch_bounds__(OS_THREADS, 1)
outer_sweep_kernel(const float* __restrict__ Wk, const float* __restrict__ U, int64_t m, int64_t d,
                   int64_t gsz, int64_t ob0, int nblk, float maxqf, uint8_t* __restrict__ codes,
                   __half* __restrict__ scales, uint8_t* __restrict__ zeros,
                   float* __restrict__ Eh_out, float* __restrict__ El_out, int64_t ldE,
                   float* __restrict__ row_loss, int first_outer, int64_t ws_stride,
                   int64_t u_stride)
{
    // matrix blockIdx.y of a batch: working copy and errors ws_stride floats
    // apart, U u_stride floats apart, the outputs packed one after the other
    {
        const int64_t e = blockIdx.y;
        Wk += e * ws_stride;
        Eh_out += e * ws_stride;
        El_out += e * ws_stride;
        U += e * u_stride;
        codes += e * m * d;
        scales += e * m * (d / gsz);
        zeros += e * m * (d / gsz);
        if (row_loss) row_loss += e * m;
    }
    extern __shared__ __align__(16) float smem[];
    float* Ws = smem;
    float* Dt = Ws + SW_ROWS * OS_WLD;
    float* rdiag = Dt + SW_B * SW_B;
    float* H0 = Dt + OS_DBUF;                  // half buffer i at H0 + i * OS_HALF
    float* Es = H0 + 2 * OS_HALF;
    const int tid = threadIdx.x;
    const bool sweeper = tid < SW_THREADS;
    const int64_t r0 = int64_t(blockIdx.x) * SW_ROWS;
    {
        const int ncol4 = nblk * SW_B / 4;
        for (int i = tid; i < SW_ROWS * ncol4; i += OS_THREADS) {
            const int rr = i / ncol4, c4 = i - rr * ncol4;
            float* dst = Ws + rr * OS_WLD + 4 * c4;
            if (r0 + rr < m)
                cp_async16(dst, Wk + (r0 + rr) * d + ob0 + 4 * c4);
            else
                *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        os_copy_diag(U, d, ob0, Dt, tid, OS_THREADS);
        cp_async_commit();
        cp_async_wait_all();
    }
    __syncthreads();
    if (tid < SW_B) {
        const int f = tid / 4;
        rdiag[tid] = 1.0f / Dt[tid * SW_B + ((f % SW_Q4) * SW_LPR + f / SW_Q4) * 4 + tid % 4];
    }
    __syncthreads();

    // sweep warps: rows of each lane (sweep_core's mapping)
    const int lane = tid & 31, sub = lane & (SW_LPR - 1);
    const int src_base = lane & ~(SW_LPR - 1);
    const int lbase = ((tid & (SW_THREADS - 1)) >> 5) * (32 / SW_LPR * SW_RPL) + lane / SW_LPR;
    int lr[SW_RPL];
    int64_t row[SW_RPL];
    bool valid[SW_RPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) {
        lr[r] = lbase + (32 / SW_LPR) * r;
        row[r] = r0 + lr[r];
        valid[r] = row[r] < m;
    }
    const int64_t G = d / gsz;
    float tot[SW_RPL];
#pragma unroll
    for (int r = 0; r < SW_RPL; ++r) tot[r] = 0.f;
    float Ev[SW_RPL][SW_CPL];

#pragma unroll 1
    for (int b = 0; b < nblk; ++b) {
        const int64_t j0 = ob0 + int64_t(b) * SW_B;
        // ---- phase A: sweep block b || block b-1's errors onto blocks b+1 ..
        if (sweeper) {
            float w[SW_RPL][SW_CPL];
#pragma unroll
            for (int r = 0; r < SW_RPL; ++r) {
                const float4* p = reinterpret_cast<const float4*>(Ws + lr[r] * OS_WLD + b * SW_B +
                                                                  SW_CPL * sub);
#pragma unroll
                for (int q = 0; q < SW_Q4; ++q) {
                    const float4 v = p[q];
                    w[r][4 * q] = v.x; w[r][4 * q + 1] = v.y; w[r][4 * q + 2] = v.z; w[r][4 * q + 3] = v.w;
                }
            }
            uint32_t cp[SW_RPL][SW_Q4];
            float loss[SW_RPL];
            sweep_core<GS, STATIC>(Dt, rdiag, w, row, valid, sub, src_base, G, gsz, j0, maxqf,
                                   scales, zeros, Ev, cp, loss);
#pragma unroll
            for (int r = 0; r < SW_RPL; ++r) {
                tot[r] += loss[r];
                if (!valid[r]) continue;
#pragma unroll
                for (int u = 0; u < SW_CPL / 16; ++u)
                    *reinterpret_cast<uint4*>(codes + row[r] * d + j0 + SW_CPL * sub + 16 * u) =
                        make_uint4(cp[r][4 * u], cp[r][4 * u + 1], cp[r][4 * u + 2], cp[r][4 * u + 3]);
                float4* hdst = reinterpret_cast<float4*>(Eh_out + row[r] * ldE + b * SW_B + SW_CPL * sub);
                float4* ldst = reinterpret_cast<float4*>(El_out + row[r] * ldE + b * SW_B + SW_CPL * sub);
#pragma unroll
                for (int q = 0; q < SW_Q4; ++q) {
                    float4 h, l;
                    h.x = tf32_round(Ev[r][4 * q + 0]); l.x = Ev[r][4 * q + 0] - h.x;
                    h.y = tf32_round(Ev[r][4 * q + 1]); l.y = Ev[r][4 * q + 1] - h.y;
                    h.z = tf32_round(Ev[r][4 * q + 2]); l.z = Ev[r][4 * q + 2] - h.z;
                    h.w = tf32_round(Ev[r][4 * q + 3]); l.w = Ev[r][4 * q + 3] - h.w;
                    hdst[q] = h;
                    ldst[q] = l;
                }
            }
        } else {
            const int ut = tid - SW_THREADS;
            const int c0w = 32 * (ut >> 5);                     // this warp's 32 columns
            const int nh = (b >= 1) ? 2 * (nblk - 1 - b) : 0;   // halves of E_{b-1}'s tiles
            const int64_t kb = j0 - SW_B;                       // U rows of block b-1
            if (nh > 0) os_copy_half(U, d, kb, j0 + SW_B, H0, ut, SW_THREADS);
            cp_async_commit();
            float acc[2][4][4];
#pragma unroll 1
            for (int h = 0; h < nh; ++h) {
                const int b2 = b + 1 + h / 2, kh = h & 1;
                if (h + 1 < nh)
                    os_copy_half(U, d, kb + ((h + 1) & 1) * (SW_B / 2),
                                 ob0 + int64_t(b + 1 + (h + 1) / 2) * SW_B,
                                 H0 + ((h + 1) & 1) * OS_HALF, ut, SW_THREADS);
                cp_async_commit();
                cp_async_wait_all_but_newest();
                bar_named(1, SW_THREADS);        // half h landed for every update thread
                if (kh == 0) {
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                            for (int v = 0; v < 4; ++v) acc[mt][nt][v] = 0.f;
                }
                os_mma_half<4>(acc, Es, H0 + (h & 1) * OS_HALF, kh * (SW_B / 2), c0w, lane);
                if (kh == 1) os_mma_subtract<4>(Ws, b2, acc, c0w, lane);
                bar_named(1, SW_THREADS);        // buffer h & 1 free
            }
            // phase B's tile (block b's rows, block b+1's columns), copied ahead
            if (b + 1 < nblk) {
                os_copy_half(U, d, j0, j0 + SW_B, H0, ut, SW_THREADS);
                os_copy_half(U, d, j0 + SW_B / 2, j0 + SW_B, H0 + OS_HALF, ut, SW_THREADS);
            }
            cp_async_commit();
        }
        __syncthreads();                         // block b swept; E_{b-1} applied
        if (b + 1 < nblk) {
            // ---- phase B: block b's errors onto block b+1, every warp
            if (sweeper) {
#pragma unroll
                for (int r = 0; r < SW_RPL; ++r)
#pragma unroll
                    for (int q = 0; q < SW_Q4; ++q)
                        *reinterpret_cast<float4*>(Es + lr[r] * OS_ELD + SW_CPL * sub + 4 * q) =
                            make_float4(Ev[r][4 * q], Ev[r][4 * q + 1], Ev[r][4 * q + 2],
                                        Ev[r][4 * q + 3]);
                os_copy_diag(U, d, j0 + SW_B, Dt, tid, SW_THREADS);
                cp_async_commit();
            } else {
                cp_async_wait_all();             // phase B's tile
            }
            __syncthreads();                     // E_b and the tile visible
            {
                const int c0w = 16 * (tid >> 5);                // this warp's 16 columns
                float acc[2][2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int v = 0; v < 4; ++v) acc[mt][nt][v] = 0.f;
                os_mma_half<2>(acc, Es, H0, 0, c0w, lane);
                os_mma_half<2>(acc, Es, H0 + OS_HALF, SW_B / 2, c0w, lane);
                os_mma_subtract<2>(Ws, b + 1, acc, c0w, lane);
            }
            if (sweeper) cp_async_wait_all();    // the next diagonal tile
            __syncthreads();
            if (tid < SW_B) {
                const int f = tid / 4;
                rdiag[tid] = 1.0f / Dt[tid * SW_B + ((f % SW_Q4) * SW_LPR + f / SW_Q4) * 4 + tid % 4];
            }
            __syncthreads();
        }
    }
    if (sweeper && row_loss && sub == 0) {
#pragma unroll
        for (int r = 0; r < SW_RPL; ++r)
            if (valid[r]) row_loss[row[r]] = first_outer ? tot[r] : row_loss[row[r]] + tot[r];
    }
}

// Round-to-nearest: one warp per (row, 128-column segment), 4 columns per lane.
template <int GS, typename T>
__global__ void __launch_bounds__(256)
rtn_kernel(const T* __restrict__ W, int64_t m, int64_t d, float maxqf,
           uint8_t* __restrict__ codes, __half* __restrict__ scales, uint8_t* __restrict__ zeros)
{
    const int64_t seg = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t segs_per_row = d / 128;
    if (seg >= m * segs_per_row) return;   // whole warp exits together
    const int64_t row = seg / segs_per_row;
    const int64_t c0 = (seg - row * segs_per_row) * 128 + 4 * lane;
    float x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) x[q] = float(W[row * d + c0 + q]);
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) { mn = fminf(mn, x[q]); mx = fmaxf(mx, x[q]); }
#pragma unroll
    for (int o = 1; o < GS / 4; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    }
    const GroupQ gq = group_params(mn, mx, maxqf);
    uint32_t packed = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) packed |= uint32_t(quant_code(x[q], gq, maxqf)) << (8 * q);
    *reinterpret_cast<uint32_t*>(codes + row * d + c0) = packed;
    if ((lane % (GS / 4)) == 0) {
        const int64_t G = d / GS;
        const int64_t gi = c0 / GS;
        scales[row * G + gi] = gq.h;
        zeros[row * G + gi] = (uint8_t)gq.z;
    }
}

// Group parameters from the working copy: one warp per (row, group) for the
// groups g_first .. g_first + g_count - 1; min/max over the group with the
// range including 0, then the same group_params as the sweep and RTN.
// Called on the uncorrected copy for static groups (all groups at once), or
// at a wide dynamic group's first column, when every column of the group has
// received every earlier column's correction (see quantize_impl).
__global__ void __launch_bounds__(256)
static_params_kernel(const float* __restrict__ Wk, int64_t m, int64_t d, int64_t gsz,
                     int64_t g_first, int64_t g_count, float maxqf, __half* __restrict__ scales,
                     uint8_t* __restrict__ zeros)
{
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t G = d / gsz;
    if (wid >= m * g_count) return;         // whole warp exits together
    const int64_t row = wid / g_count, gi = g_first + (wid - row * g_count);
    const float* p = Wk + row * d + gi * gsz;
    float mn = 0.f, mx = 0.f;
    for (int64_t c = 4 * lane; c < gsz; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(p + c);
        mn = fminf(fminf(mn, v.x), fminf(v.y, fminf(v.z, v.w)));
        mx = fmaxf(fmaxf(mx, v.x), fmaxf(v.y, fmaxf(v.z, v.w)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    }
    if (lane == 0) {
        const GroupQ gq = group_params(mn, mx, maxqf);
        scales[row * G + gi] = gq.h;
        zeros[row * G + gi] = (uint8_t)gq.z;
    }
}

// Round-to-nearest for groups wider than 128 columns (or one group per
// row): one warp per (row, group), min/max in a first pass over the group,
// the codes in a second.
template <typename T>
__global__ void __launch_bounds__(256)
rtn_wide_kernel(const T* __restrict__ W, int64_t m, int64_t d, int64_t gsz, float maxqf,
                uint8_t* __restrict__ codes, __half* __restrict__ scales,
                uint8_t* __restrict__ zeros)
{
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t G = d / gsz;
    if (wid >= m * G) return;               // whole warp exits together
    const int64_t row = wid / G, gi = wid - row * G;
    const T* p = W + row * d + gi * gsz;
    float mn = 0.f, mx = 0.f;
    for (int64_t c = 4 * lane; c < gsz; c += 128) {
#pragma unroll
        for (int q = 0; q < 4; ++q) { const float x = float(p[c + q]); mn = fminf(mn, x); mx = fmaxf(mx, x); }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    }
    const GroupQ gq = group_params(mn, mx, maxqf);
    for (int64_t c = 4 * lane; c < gsz; c += 128) {
        uint32_t packed = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) packed |= uint32_t(quant_code(float(p[c + q]), gq, maxqf)) << (8 * q);
        *reinterpret_cast<uint32_t*>(codes + row * d + gi * gsz + c) = packed;
    }
    if (lane == 0) {
        scales[row * G + gi] = gq.h;
        zeros[row * G + gi] = (uint8_t)gq.z;
    }
}

struct QuantWs {
    float* Wk;     // d_out x d_in working copy (sweep order)
    UpdateWs upd;  // split U and the current block's split errors
};

static size_t quant_layout(int64_t m, int64_t d, char* base, QuantWs* w)
{
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 1024); return o; };
    size_t oW = take(sizeof(float) * m * d);
    size_t oU = take(update_ws_bytes(m, d));
    if (w && base) {
        w->Wk = reinterpret_cast<float*>(base + oW);
        update_ws_bind(m, d, base + oU, &w->upd);
    }
    return off;
}

static int check_quant_args(int w_dtype, int64_t m, int64_t d, int bits)
{
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_INVALID_ARG;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return GPTQ_ERR_UNSUPPORTED;
    if (d < 128 || d > kMaxDim || d % 128 != 0) return GPTQ_ERR_SHAPE;
    if (m < 1 || m > kMaxRows) return GPTQ_ERR_SHAPE;
    return GPTQ_OK;
}

template <int GS, bool STATIC>
static void launch_sweep(dim3 grid, size_t smem, cudaStream_t st, const float* Wk, const float* U,
                         int64_t m, int64_t d, int64_t gsz, int64_t j0, float maxqf,
                         uint8_t* codes, __half* scales, uint8_t* zeros, float* Eh, float* El,
                         int64_t ldE, float* row_loss, int first)
{
    cudaFuncSetAttribute(block_sweep_kernel<GS, STATIC>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    KernelTimer kt(kKSweep, st);
    block_sweep_kernel<GS, STATIC><<<grid, SW_THREADS, smem, st>>>(
        Wk, U, m, d, gsz, j0, maxqf, codes, scales, zeros, Eh, El, ldE, row_loss, first);
    count_launches();
}

template <int GS, bool STATIC>
static void launch_outer(dim3 grid, cudaStream_t st, const float* Wk, const float* U, int64_t m,
                         int64_t d, int64_t gsz, int64_t ob0, int nblk, float maxqf,
                         uint8_t* codes, __half* scales, uint8_t* zeros, float* Eh, float* El,
                         int64_t ldE, float* row_loss, int first, int64_t ws_stride,
                         int64_t u_stride)
{
    cudaFuncSetAttribute(outer_sweep_kernel<GS, STATIC>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OS_SMEM);
    KernelTimer kt(kKSweep, st);
    outer_sweep_kernel<GS, STATIC><<<grid, OS_THREADS, OS_SMEM, st>>>(
        Wk, U, m, d, gsz, ob0, nblk, maxqf, codes, scales, zeros, Eh, El, ldE, row_loss, first,
        ws_stride, u_stride);
    count_launches();
}

}  // namespace gptq

extern "C" size_t gptq_quantize_workspace_bytes(int64_t d_out, int64_t d_in, int block_size)
{
    if (d_out <= 0 || d_in <= 0 || block_size != gptq::SW_B) return 0;
    return gptq::quant_layout(d_out, d_in, nullptr, nullptr);
}

namespace gptq {

// Group sizes the sweep takes.  Dynamic groups (parameters at each group's
// first column from the corrected row): 32, 64, 128, and the multiples of
// 128 dividing d that either divide the 512-column outer block or are
// multiples of it -- those groups never straddle an outer-block boundary
// from the inside, so at a group's first column every column of the group
// has received every earlier column's correction (the near updates cover
// the rest of the outer block, the far updates everything beyond a finished
// outer block) and the parameters can be taken from the working copy there.
// Static groups (parameters from the rows before the sweep): 32, 64 or any
// multiple of 128 dividing d.  One group per row (-1 or d) is the same in
// both readings, since at column 0 no correction has happened yet.
static int sweep_group_size(int64_t d, int group_size, bool static_groups, int64_t* gsz)
{
    if (group_size == -1 || group_size == d) { *gsz = d; return GPTQ_OK; }
    if (group_size == 32 || group_size == 64 || group_size == 128) { *gsz = group_size; return GPTQ_OK; }
    const int64_t ob = int64_t(UPD_OUTER) * SW_B;
    if (group_size > 128 && group_size % 128 == 0 && d % group_size == 0 &&
        (static_groups || ob % group_size == 0 || group_size % ob == 0)) {
        *gsz = group_size;
        return GPTQ_OK;
    }
    return GPTQ_ERR_UNSUPPORTED;
}

// Argument checks of a layer quantization; the group mode on success.
static int quantize_checks(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                           const float* U, const int32_t* perm, int bits, int group_size,
                           int block_size, const uint8_t* codes, const uint16_t* scales,
                           const uint8_t* zeros, const float* row_loss, const void* ws,
                           size_t ws_bytes, bool static_groups, int64_t* gsz, bool* wide,
                           bool* stat)
{
    if (!W || !U || !codes || !scales || !zeros || !ws) return GPTQ_ERR_INVALID_ARG;
    int rc = check_quant_args(w_dtype, d_out, d_in, bits);
    if (rc != GPTQ_OK) return rc;
    rc = sweep_group_size(d_in, group_size, static_groups, gsz);
    if (rc != GPTQ_OK) return rc;
    // the sweep reads the group parameters instead of reducing them when they
    // are static, one per row, or dynamic but wider than a block (taken just
    // in time at each group's first block by static_params_kernel)
    *wide = !static_groups && *gsz > SW_B && *gsz < d_in;
    *stat = static_groups || *gsz == d_in || *wide;
    if (block_size != SW_B) return GPTQ_ERR_UNSUPPORTED;
    if (!aligned16(W) || !aligned16(U) || !aligned16(codes) || !aligned16(scales) ||
        !aligned16(zeros) || !aligned16(ws) || (perm && !aligned16(perm)) ||
        (row_loss && !aligned16(row_loss)))
        return GPTQ_ERR_INVALID_ARG;
    if (ws_bytes < gptq_quantize_workspace_bytes(d_out, d_in, block_size))
        return GPTQ_ERR_INVALID_ARG;
    return GPTQ_OK;
}

// Per matrix, before the sweep: the fp32 working copy in sweep order, the
// group parameters when they are taken from the rows before the sweep, and
// U's TF32 split for the tensor-core updates.
static int quantize_prepare(const void* W, int w_dtype, int64_t m, int64_t d, const float* U,
                            const int32_t* perm, int64_t gsz, bool stat, bool wide, float maxqf,
                            __half* sc, uint8_t* zeros, QuantWs& w, cudaStream_t st)
{
    {
        const int64_t total = m * d;
        const unsigned grid = (unsigned)std::min<int64_t>(ceil_div(total, 256), 148 * 16);
        KernelTimer kt(kKInitWork, st);
        if (w_dtype == GPTQ_DTYPE_F16)
            init_work_kernel<__half><<<grid, 256, 0, st>>>(reinterpret_cast<const __half*>(W), perm,
                                                           m, d, w.Wk);
        else
            init_work_kernel<float><<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(W), perm,
                                                          m, d, w.Wk);
        count_launches();
    }
    if (stat && !wide) {
        const int64_t warps = m * (d / gsz);
        KernelTimer kt(kKStaticParams, st);
        static_params_kernel<<<(unsigned)ceil_div(warps * 32, 256), 256, 0, st>>>(
            w.Wk, m, d, gsz, 0, d / gsz, maxqf, sc, zeros);
        count_launches();
    }
    KernelTimer kt(kKSplitU, st);
    return update_prepare_u(U, d, &w.upd, st);
}

// Fused outer blocks, for n_mats matrices at once (matrix e's workspace
// ws_stride bytes after matrix 0's, its U d^2 floats after, its outputs
// packed): one launch sweeps an outer block's 128-column blocks of every
// matrix and applies each block's errors to the rest of the outer block; the
// columns beyond it get the outer block's errors at once (K = 512) on the
// tensor cores.  Not for dynamic groups whose starts fall inside an outer
// block (256 columns).
static int quantize_fused(int64_t n_mats, int64_t m, int64_t d, const float* U, int64_t gsz,
                          bool stat, bool wide, float maxqf, uint8_t* codes, __half* sc,
                          uint8_t* zeros, float* row_loss, char* ws0, size_t ws_stride,
                          cudaStream_t st)
{
    const int64_t outer = int64_t(UPD_OUTER) * SW_B;
    const int64_t G = d / gsz;
    const dim3 grid((unsigned)ceil_div(m, SW_ROWS), (unsigned)n_mats);
    QuantWs w0;
    quant_layout(m, d, ws0, &w0);
    for (int64_t ob0 = 0; ob0 < d; ob0 += outer) {
        const int64_t ob1 = std::min<int64_t>(d, ob0 + outer);
        const int nb = (int)((ob1 - ob0) / SW_B);
        if (wide && ob0 % gsz == 0) {            // a wide dynamic group starts here
            for (int64_t e = 0; e < n_mats; ++e) {
                QuantWs w;
                quant_layout(m, d, ws0 + e * ws_stride, &w);
                KernelTimer kt(kKStaticParams, st);
                static_params_kernel<<<(unsigned)ceil_div(m * 32, 256), 256, 0, st>>>(
                    w.Wk, m, d, gsz, ob0 / gsz, 1, maxqf, sc + e * m * G, zeros + e * m * G);
                count_launches();
            }
        }
#define GPTQ_OUTER(GSV, STAT)                                                                   \
        launch_outer<GSV, STAT>(grid, st, w0.Wk, U, m, d, gsz, ob0, nb, maxqf, codes, sc, zeros, \
                                w0.upd.Eh, w0.upd.El, UPD_LDE, row_loss, ob0 == 0,               \
                                int64_t(ws_stride / sizeof(float)), d * d)
        if (stat) {
            switch (gsz) {
                case 32: GPTQ_OUTER(32, true); break;
                case 64: GPTQ_OUTER(64, true); break;
                default: GPTQ_OUTER(128, true); break;
            }
        } else {
            switch (gsz) {
                case 32: GPTQ_OUTER(32, false); break;
                case 64: GPTQ_OUTER(64, false); break;
                default: GPTQ_OUTER(128, false); break;
            }
        }
#undef GPTQ_OUTER
        if (ob1 < d) {
            for (int64_t e = 0; e < n_mats; ++e) {
                QuantWs w;
                quant_layout(m, d, ws0 + e * ws_stride, &w);
                KernelTimer kt(kKUpdateFar, st);
                const int rc = block_update(w.Wk, &w.upd, m, d, /*e_col0=*/0, /*k_rows=*/ob1 - ob0,
                                           /*u_row0=*/ob0, /*c_begin=*/ob1, /*c_end=*/d, st);
                if (rc != GPTQ_OK) return rc;
            }
        }
    }
    return launch_status();
}

static int quantize_impl(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                         const float* U, const int32_t* perm, int bits, int group_size,
                         int block_size, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                         float* row_loss, void* ws, size_t ws_bytes, void* stream,
                         bool static_groups)
{
    int64_t gsz = 0;
    bool wide = false, stat = false;
    int rc = quantize_checks(W, w_dtype, d_out, d_in, U, perm, bits, group_size, block_size, codes,
                             scales, zeros, row_loss, ws, ws_bytes, static_groups, &gsz, &wide,
                             &stat);
    if (rc != GPTQ_OK) return rc;
    cudaStream_t st = as_stream(stream);
    QuantWs w;
    quant_layout(d_out, d_in, reinterpret_cast<char*>(ws), &w);
    const int64_t m = d_out, d = d_in;
    const float maxqf = float((1 << bits) - 1);
    __half* sc = reinterpret_cast<__half*>(scales);
    rc = quantize_prepare(W, w_dtype, m, d, U, perm, gsz, stat, wide, maxqf, sc, zeros, w, st);
    if (rc != GPTQ_OK) return rc;
    const int64_t outer = int64_t(UPD_OUTER) * SW_B;
    if (!wide || gsz % outer == 0)
        return quantize_fused(1, m, d, U, gsz, stat, wide, maxqf, codes, sc, zeros, row_loss,
                              reinterpret_cast<char*>(ws), 0, st);
    // Dynamic groups of 256 columns: a sweep launch per 128-column block, the
    // rest of the outer block updated after each (K = 128), the columns
    // beyond an outer block after its last block (K = 512).  Every column
    // still receives every earlier column's correction before its own block
    // is swept.
    const dim3 grid((unsigned)ceil_div(m, SW_ROWS));
    const size_t smem = sizeof(float) * (SW_B * SW_B + SW_B);
    const int64_t nblk = d / SW_B;
    for (int64_t b = 0; b < nblk; ++b) {
        const int64_t j0 = b * SW_B;
        const int64_t ob0 = (b / UPD_OUTER) * UPD_OUTER * SW_B;            // outer block start
        const int64_t ob1 = std::min<int64_t>(d, ob0 + UPD_OUTER * SW_B);  // and end
        const int64_t ecol = j0 - ob0;                                     // E column of this block
        float* Eh = w.upd.Eh + ecol;
        float* El = w.upd.El + ecol;
        if (wide && j0 % gsz == 0) {            // a wide dynamic group starts here
            KernelTimer kt(kKStaticParams, st);
            static_params_kernel<<<(unsigned)ceil_div(m * 32, 256), 256, 0, st>>>(
                w.Wk, m, d, gsz, j0 / gsz, 1, maxqf, sc, zeros);
            count_launches();
        }
#define GPTQ_SWEEP(GSV, STAT)                                                                   \
        launch_sweep<GSV, STAT>(grid, smem, st, w.Wk, U, m, d, gsz, j0, maxqf, codes, sc, zeros, \
                                Eh, El, UPD_LDE, row_loss, b == 0)
        if (stat) {
            switch (gsz) {
                case 32: GPTQ_SWEEP(32, true); break;
                case 64: GPTQ_SWEEP(64, true); break;
                default: GPTQ_SWEEP(128, true); break;     // groups of 128 or more
            }
        } else {
            switch (gsz) {
                case 32: GPTQ_SWEEP(32, false); break;
                case 64: GPTQ_SWEEP(64, false); break;
                default: GPTQ_SWEEP(128, false); break;
            }
        }
#undef GPTQ_SWEEP
        if (j0 + SW_B < ob1) {                                   // near: rest of the outer block
            KernelTimer kt(kKUpdateNear, st);
            rc = block_update(w.Wk, &w.upd, m, d, /*e_col0=*/ecol, /*k_rows=*/SW_B, /*u_row0=*/j0,
                              /*c_begin=*/j0 + SW_B, /*c_end=*/ob1, st);
            if (rc != GPTQ_OK) return rc;
        }
        if (j0 + SW_B == ob1 && ob1 < d) {                       // far: everything beyond it
            KernelTimer kt(kKUpdateFar, st);
            rc = block_update(w.Wk, &w.upd, m, d, /*e_col0=*/0, /*k_rows=*/ob1 - ob0,
                              /*u_row0=*/ob0, /*c_begin=*/ob1, /*c_end=*/d, st);
            if (rc != GPTQ_OK) return rc;
        }
    }
    return launch_status();
}

}  // namespace gptq

extern "C" int gptq_quantize_layer(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                                   const float* U, const int32_t* perm, int bits, int group_size,
                                   int block_size, uint8_t* codes, uint16_t* scales,
                                   uint8_t* zeros, float* row_loss, void* ws, size_t ws_bytes,
                                   void* stream)
{
    return gptq::quantize_impl(W, w_dtype, d_out, d_in, U, perm, bits, group_size, block_size,
                               codes, scales, zeros, row_loss, ws, ws_bytes, stream, false);
}

extern "C" int gptq_quantize_layer_static(const void* W, int w_dtype, int64_t d_out,
                                          int64_t d_in, const float* U, const int32_t* perm,
                                          int bits, int group_size, int block_size,
                                          uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                                          float* row_loss, void* ws, size_t ws_bytes,
                                          void* stream)
{
    return gptq::quantize_impl(W, w_dtype, d_out, d_in, U, perm, bits, group_size, block_size,
                               codes, scales, zeros, row_loss, ws, ws_bytes, stream, true);
}

extern "C" int gptq_quantize_layer_batched(const void* W, int w_dtype, int64_t n_mats,
                                           int64_t d_out, int64_t d_in, const float* U,
                                           const int32_t* perm, int bits, int group_size,
                                           int block_size, uint8_t* codes, uint16_t* scales,
                                           uint8_t* zeros, float* row_loss, void* ws,
                                           size_t ws_bytes, void* stream)
{
    using namespace gptq;
    if (n_mats < 1 || n_mats > 4096) return GPTQ_ERR_SHAPE;
    if (!W || !U || !codes || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
    int64_t gsz = 0;
    int rc = sweep_group_size(d_in, group_size, false, &gsz);
    if (rc != GPTQ_OK) return rc;
    const int64_t G = d_in / gsz;
    const size_t wb = (w_dtype == GPTQ_DTYPE_F16) ? 2 : 4;
    // every matrix's arrays must stay 16-byte aligned at their offsets
    if ((d_out * d_in * int64_t(wb)) % 16 || (d_out * G * 2) % 16 || (d_out * G) % 16 ||
        (row_loss && (d_out * 4) % 16) || (perm && (d_in * 4) % 16))
        return GPTQ_ERR_SHAPE;
    // With a workspace per matrix (n_mats times the single-matrix size), every
    // outer block is one fused launch over all the matrices (their row tiles
    // fill the SMs' waves together) followed by each matrix's far update;
    // otherwise one matrix after the other shares the one workspace.
    const size_t single = gptq_quantize_workspace_bytes(d_out, d_in, block_size);
    if (n_mats > 1 && single > 0 && ws && ws_bytes / size_t(n_mats) >= single) {
        bool wide = false, stat = false;
        int64_t g2 = 0;
        rc = quantize_checks(W, w_dtype, d_out, d_in, U, perm, bits, group_size, block_size,
                             codes, scales, zeros, row_loss, ws, single, false, &g2, &wide, &stat);
        if (rc != GPTQ_OK) return rc;
        if (!wide || g2 % (int64_t(UPD_OUTER) * SW_B) == 0) {
            cudaStream_t st = as_stream(stream);
            const float maxqf = float((1 << bits) - 1);
            __half* sc = reinterpret_cast<__half*>(scales);
            char* ws0 = reinterpret_cast<char*>(ws);
            for (int64_t e = 0; e < n_mats; ++e) {
                QuantWs w;
                quant_layout(d_out, d_in, ws0 + e * single, &w);
                rc = quantize_prepare(reinterpret_cast<const char*>(W) + e * d_out * d_in * int64_t(wb),
                                      w_dtype, d_out, d_in, U + e * d_in * d_in,
                                      perm ? perm + e * d_in : nullptr, g2, stat, wide, maxqf,
                                      sc + e * d_out * G, zeros + e * d_out * G, w, st);
                if (rc != GPTQ_OK) return rc;
            }
            return quantize_fused(n_mats, d_out, d_in, U, g2, stat, wide, maxqf, codes, sc, zeros,
                                  row_loss, ws0, single, st);
        }
    }
    for (int64_t e = 0; e < n_mats; ++e) {
        rc = quantize_impl(reinterpret_cast<const char*>(W) + e * d_out * d_in * int64_t(wb),
                           w_dtype, d_out, d_in, U + e * d_in * d_in,
                           perm ? perm + e * d_in : nullptr, bits, group_size, block_size,
                           codes + e * d_out * d_in, scales + e * d_out * G, zeros + e * d_out * G,
                           row_loss ? row_loss + e * d_out : nullptr, ws, ws_bytes, stream, false);
        if (rc != GPTQ_OK) return rc;
    }
    return GPTQ_OK;
}

extern "C" int rtn_quantize(const void* W, int w_dtype, int64_t d_out, int64_t d_in, int bits,
                            int group_size, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                            void* stream)
{
    using namespace gptq;
    if (!W || !codes || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
    int rc = check_quant_args(w_dtype, d_out, d_in, bits);
    if (rc != GPTQ_OK) return rc;
    const int64_t gsz = (group_size == -1) ? d_in : group_size;
    const bool narrow = gsz == 32 || gsz == 64 || gsz == 128;
    if (!narrow && !(gsz > 128 && gsz % 128 == 0 && d_in % gsz == 0)) return GPTQ_ERR_UNSUPPORTED;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros))
        return GPTQ_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    const float maxqf = float((1 << bits) - 1);
    if (!narrow) {
        const int64_t warps = d_out * (d_in / gsz);
        const unsigned grid = (unsigned)ceil_div(warps * 32, 256);
        __half* sc = reinterpret_cast<__half*>(scales);
        KernelTimer kt(kKRtn, st);
        if (w_dtype == GPTQ_DTYPE_F16)
            rtn_wide_kernel<__half><<<grid, 256, 0, st>>>(reinterpret_cast<const __half*>(W),
                                                          d_out, d_in, gsz, maxqf, codes, sc,
                                                          zeros);
        else
            rtn_wide_kernel<float><<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(W), d_out,
                                                         d_in, gsz, maxqf, codes, sc, zeros);
        count_launches();
        return launch_status();
    }
    const int64_t warps = d_out * (d_in / 128);
    const unsigned grid = (unsigned)ceil_div(warps * 32, 256);
    __half* sc = reinterpret_cast<__half*>(scales);
    KernelTimer kt(kKRtn, st);
#define GPTQ_RTN_LAUNCH(GSV)                                                                     \
    if (w_dtype == GPTQ_DTYPE_F16)                                                               \
        rtn_kernel<GSV, __half><<<grid, 256, 0, st>>>(reinterpret_cast<const __half*>(W), d_out, \
                                                      d_in, maxqf, codes, sc, zeros);            \
    else                                                                                         \
        rtn_kernel<GSV, float><<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(W), d_out,   \
                                                     d_in, maxqf, codes, sc, zeros);
    switch (group_size) {
        case 32: GPTQ_RTN_LAUNCH(32) break;
        case 64: GPTQ_RTN_LAUNCH(64) break;
        default: GPTQ_RTN_LAUNCH(128) break;
    }
#undef GPTQ_RTN_LAUNCH
    count_launches();
    return launch_status();
}

// Test hook: out[i] = the sweep's division-free quotient of x[i] / s[i] with
// r = RN(1 / s[i]), computed on the host by the same function the kernels
// use (FMAs are correctly rounded on both sides).
extern "C" int gptq_debug_div_rn(const float* x, const float* s, int64_t n, float* out)
{
    if (n < 0 || (n > 0 && (!x || !s || !out))) return GPTQ_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n; ++i) {
        const float r = 1.0f / s[i];
        out[i] = gptq::div_rn_recip(x[i], s[i], r);
    }
    return GPTQ_OK;
}
