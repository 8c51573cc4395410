// Several tokens through one sparse product, served from the union of their kept rows on
// the tcgen05 tensor cores (the batched form of the sparse product of "Spark Transformer",
// section 3.1; the union of the active columns of a token block is the shape that
// "Sparser, Faster, Lighter Transformer Language Models" packs for its CUDA kernels):
//
//   U        = union over the block's tokens of their kept channels (ascending);
//   X~[b][i] = xs of token b at channel U_i if token b kept it, else 0, as up to three
//              bf16 parts (x = hi + mid + lo to float32 precision; the residue parts are
//              used only when some value of the block is not exactly a bf16);
//   Y[b][:]  = sum over i of X~[b][i] * Wt[U_i][:]      (float32, tensor-core MMA),
//
// so every kept row is read from HBM once per token block, whatever the number of
// tokens that keep it. The K dimension is cut into chunks of 64 rows: a block of 64
// consecutive channels of which at least kDenseMin are in the union is one chunk, loaded
// as one 64-row TMA tile (its other rows carry zero inputs), and the members of the other
// blocks are packed 64 to a chunk and loaded by four-row TMA gathers (a gather moves 512
// bytes, a tile 8 KB, so mostly-full blocks are cheaper as tiles). The product is
// D[m][b] = A[m][i] * B[i][b] with A = the chunk's rows of Wt for a 128-output tile (128-byte
// swizzle, M-major operand) and B = X~ (K-major); D accumulates every part in tensor
// memory. CTAs take (128-output tile, range of chunks) and add their D into Y.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "tc.cuh"

namespace wina {

constexpr int kUT = 192;           // threads: warp 0 loads, warp 1 issues MMAs, warps 2-5 drain D
constexpr int kUBlock = kUnionBlock;  // tokens per block (the MMA's largest N)
constexpr int kUChunk = 64;        // union rows per pipeline stage (one 128-byte swizzle span of X~)
constexpr int kUMaxStages = 8;
constexpr int kDenseMin = 20;      // members of a 64-channel block that make it a tile chunk

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) {
  const uint32_t u = __float_as_uint(v);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// Union of the kept channels of tokens [b0, b0 + nb): flag[j] = 1 (plain byte stores;
// several tokens may store the same 1).
__global__ void k_union_mark(const int32_t* __restrict__ idx, int ld, int k, const int32_t* __restrict__ count, int n,
                             int b0, uint8_t* __restrict__ flag, int32_t* status) {
  const int b = b0 + blockIdx.x;
  const int kb = k >= 0 ? k : max(0, min(__ldg(count + b), ld));
  for (int r = threadIdx.x; r < kb; r += blockDim.x) {
    const int j = __ldg(idx + (int64_t)b * ld + r);
    if (j < 0 || j >= n) {
      record_status(status, WINA_ERR_INVALID_ARG);
      continue;
    }
    flag[j] = 1;
  }
}

// Chunk plan of the union and each member's place (one CTA of 1024 threads, n <= 65536).
// Thread q counts the members of channel block [64q, 64q + 64); blocks with at least
// kDenseMin members become tile chunks (in block order), the members of the others are
// packed into gather chunks after them. chunk_row[c] = the first channel of tile chunk c,
// -1 for a gather chunk; info[0] = chunks, info[1] = 1 (bf16 parts of X~, raised later),
// info[2] = tile chunks. Then, block by block (a warp per block), each member's X~ column
// pos[j] (its slot in a tile chunk, or its packed place in a gather chunk, whose slot then
// names it) is written and the flags are cleared for the next call. The padding slots of
// the last gather chunk point at channel 0 (their inputs are zero).
__global__ void __launch_bounds__(1024) k_union_plan(uint8_t* __restrict__ flag, int n, int32_t* __restrict__ chunk_row,
                                                     int32_t* __restrict__ slot, int32_t* __restrict__ pos,
                                                     uint32_t* __restrict__ info) {
  __shared__ uint32_t red[33];
  __shared__ int32_t s_base[1024];
  __shared__ uint8_t s_dense[1024];
  const int q = threadIdx.x;
  const int nblk = (n + 63) / 64;
  uint32_t cnt = 0;
  if (q < nblk) {
    for (int r = 0; r < 64; r += 4) {
      const int j = q * 64 + r;
      if (j < n) {
        const uint32_t w = j + 4 <= n ? *reinterpret_cast<const uint32_t*>(flag + j) : 0u;
        if (j + 4 <= n) {
          cnt += (w & 0xFFu ? 1u : 0u) + (w & 0xFF00u ? 1u : 0u) + (w & 0xFF0000u ? 1u : 0u) + (w >> 24 ? 1u : 0u);
        } else {
          for (int e = j; e < n; ++e) cnt += flag[e] ? 1u : 0u;
        }
      }
    }
  }
  const bool dense = cnt >= (uint32_t)kDenseMin;
  uint32_t ndense, ngath;
  const uint32_t di = block_excl_scan<1024>(dense ? 1u : 0u, red, &ndense);
  const uint32_t go = block_excl_scan<1024>(dense ? 0u : cnt, red, &ngath);
  if (q < nblk) {
    s_base[q] = dense ? (int32_t)(di * 64) : (int32_t)(ndense * 64 + go);
    s_dense[q] = dense ? 1 : 0;
    if (dense) chunk_row[di] = q * 64;
  }
  const uint32_t ngc = (ngath + 63) / 64;
  for (uint32_t g = q; g < ngc; g += 1024) chunk_row[ndense + g] = -1;
  for (uint32_t i = ndense * 64 + ngath + q; i < (ndense + ngc) * 64; i += 1024) slot[i] = 0;
  if (q == 0) {
    info[0] = ndense + ngc;
    info[1] = 1u;
    info[2] = ndense;
  }
  __syncthreads();
  // members' places, a warp per 64-channel block (lane l: channels 64q + l and 64q + 32 + l)
  const int warp = q >> 5, lane = q & 31;
  for (int qb = warp; qb < nblk; qb += 32) {
    const int j0 = qb * 64 + lane, j1 = j0 + 32;
    const bool f0 = j0 < n && flag[j0] != 0, f1 = j1 < n && flag[j1] != 0;
    const uint32_t b0 = __ballot_sync(0xffffffffu, f0), b1 = __ballot_sync(0xffffffffu, f1);
    if (j0 < n) flag[j0] = 0;
    if (j1 < n) flag[j1] = 0;
    const int32_t base = s_base[qb];
    const uint32_t below = (1u << lane) - 1u;
    if (s_dense[qb]) {
      if (f0) pos[j0] = base + lane;
      if (f1) pos[j1] = base + 32 + lane;
    } else {
      if (f0) {
        const int32_t p = base + (int32_t)__popc(b0 & below);
        pos[j0] = p;
        slot[p] = j0;
      }
      if (f1) {
        const int32_t p = base + (int32_t)(__popc(b0) + __popc(b1 & below));
        pos[j1] = p;
        slot[p] = j1;
      }
    }
  }
}

// X~ of tokens [b0, b0 + nb) as bf16 rows, part p (hi, mid, lo) of token b in row p * NP + b
// (row stride kmax): each kept channel's value at its column pos[j]. Every other entry of
// X~ is zero: the workspace starts zeroed and k_union_clear puts zeros back where this
// kernel wrote once the product has read them. info[1] receives the number of parts the
// block needs (1 when every value is exactly a bf16). The tokens' rows of Y (m floats
// each, m % 4 == 0) are zeroed for the product's sums. Grid: (tokens, slices of 256 kept
// entries).
__global__ void __launch_bounds__(256) k_union_xt(const int32_t* __restrict__ idx, const float* __restrict__ xs,
                                                  int ld, int k, const int32_t* __restrict__ count, int n, int b0,
                                                  int NP, const int32_t* __restrict__ pos, uint32_t* __restrict__ info,
                                                  uint16_t* __restrict__ xt, int kmax, float* __restrict__ y, int m) {
  const int rb = blockIdx.x;
  const int b = b0 + rb;
  {  // this CTA's slice of token b's row of Y
    const int m4 = m / 4;
    const int q0 = (int)((int64_t)m4 * blockIdx.y / gridDim.y), q1 = (int)((int64_t)m4 * (blockIdx.y + 1) / gridDim.y);
    float4* yr = reinterpret_cast<float4*>(y + (int64_t)b * m);
    for (int q = q0 + threadIdx.x; q < q1; q += 256) yr[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int kb = k >= 0 ? k : max(0, min(__ldg(count + b), ld));
  uint32_t need = 1u;
  const int r = blockIdx.y * 256 + threadIdx.x;
  if (r < kb) {
    const int j = __ldg(idx + (int64_t)b * ld + r);
    if (j >= 0 && j < n) {  // out-of-range entries are reported by the marking
      const float v = __ldg(xs + (int64_t)b * ld + r);
      // v = hi + mid + lo + (a residue below float32 resolution); each difference is exact
      const uint16_t h = bf16_rn_bits(v);
      const float r1 = v - __uint_as_float((uint32_t)h << 16);
      const uint16_t md = bf16_rn_bits(r1);
      const float r2 = r1 - __uint_as_float((uint32_t)md << 16);
      const uint16_t l = bf16_rn_bits(r2);
      const int p = pos[j];
      xt[(size_t)rb * kmax + p] = h;
      xt[((size_t)NP + rb) * kmax + p] = md;
      xt[((size_t)2 * NP + rb) * kmax + p] = l;
      need = (l & 0x7FFFu) ? 3u : ((md & 0x7FFFu) ? 2u : 1u);
    }
  }
  need = __reduce_max_sync(0xffffffffu, need);
  if ((threadIdx.x & 31) == 0 && need > 1u) atomicMax(info + 1, need);
}

// Zeros back into the entries of X~ that k_union_xt wrote (same grid), after the product.
__global__ void __launch_bounds__(256) k_union_clear(const int32_t* __restrict__ idx, int ld, int k,
                                                     const int32_t* __restrict__ count, int n, int b0, int NP,
                                                     const int32_t* __restrict__ pos, uint16_t* __restrict__ xt,
                                                     int kmax) {
  const int rb = blockIdx.x;
  const int b = b0 + rb;
  const int kb = k >= 0 ? k : max(0, min(__ldg(count + b), ld));
  const int r = blockIdx.y * 256 + threadIdx.x;
  if (r < kb) {
    const int j = __ldg(idx + (int64_t)b * ld + r);
    if (j >= 0 && j < n) {
      const int p = pos[j];
      xt[(size_t)rb * kmax + p] = 0;
      xt[((size_t)NP + rb) * kmax + p] = 0;
      xt[((size_t)2 * NP + rb) * kmax + p] = 0;
    }
  }
}

// Y[b0 + b][m0 .. m0 + 127] += D for this CTA's chunks of U. Grid: (m tiles) x (K splits).
__global__ void __launch_bounds__(kUT, 1)
    k_union_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmT,
                 const __grid_constant__ CUtensorMap tmX, const int32_t* __restrict__ chunk_row,
                 const int32_t* __restrict__ slot, const uint32_t* __restrict__ info, int m, int nb, int NP,
                 int ksplit, float* __restrict__ y, int b0, int smem_bytes, int32_t* status) {
  extern __shared__ unsigned char smraw[];
  __shared__ uint64_t full[kUMaxStages], empty[kUMaxStages], done;
  __shared__ uint32_t s_taddr;
  __shared__ int s_abort;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int mt = blockIdx.x % ((m + 127) / 128), ks = blockIdx.x / ((m + 127) / 128);
  const int m0 = mt * 128;
  const int nch = (int)info[0];
  const int c0 = (int)((int64_t)nch * ks / ksplit), c1 = (int)((int64_t)nch * (ks + 1) / ksplit);
  if (c0 >= c1) return;  // nothing for this CTA (uniform)
  const int P = (int)min(3u, max(1u, info[1]));  // bf16 parts of X~
  // stage layout: A (two 64-output boxes of 64 rows x 128 B) | X~ parts (NP rows x 128 B each)
  const uint32_t sbase = (tc::smem_u32(smraw) + 1023u) & ~1023u;
  unsigned char* gbase = smraw + (sbase - tc::smem_u32(smraw));
  const uint32_t a_bytes = 2u * kUChunk * 128u, x_bytes = (uint32_t)NP * 128u;
  const uint32_t stage_bytes = (a_bytes + x_bytes * (uint32_t)P + 1023u) & ~1023u;
  int S = (int)(((uint32_t)smem_bytes - 1024u) / stage_bytes);
  S = S > kUMaxStages ? kUMaxStages : S;
  const uint32_t ncols = NP <= 32 ? 32u : (NP <= 64 ? 64u : (NP <= 128 ? 128u : 256u));
  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full[s], 1u);
      tc::mbar_init(&empty[s], 1u);
    }
    tc::mbar_init(&done, 1u);
    tc::mbar_init_fence();
    s_abort = 0;
  }
  if (warp == 2) tc::tmem_alloc(&s_taddr, ncols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t taddr = s_taddr;

  if (warp == 0) {
    // ---------------- loads: X~ tiles; A as two 64-row tiles or 16 four-row gathers ----------------
    const uint32_t bytes = a_bytes + x_bytes * (uint32_t)P;
    int issued = 0;
    int32_t row0 = chunk_row[c0];
    int32_t u0 = row0 < 0 ? slot[c0 * kUChunk + lane] : 0, u1 = row0 < 0 ? slot[c0 * kUChunk + 32 + lane] : 0;
    for (int c = c0; c < c1; ++c) {
      const int it = c - c0, s = it % S;
      // the next chunk's rows are read while this one's stage frees
      int32_t nrow = 0, n0 = 0, n1 = 0;
      if (c + 1 < c1) {
        nrow = chunk_row[c + 1];
        if (nrow < 0) {
          n0 = slot[(c + 1) * kUChunk + lane];
          n1 = slot[(c + 1) * kUChunk + 32 + lane];
        }
      }
      bool ok = true;
      if (lane == 0 && it >= S) ok = tc::mbar_wait(&empty[s], (uint32_t)((it / S - 1) & 1));
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok || *(volatile int*)&s_abort) {
        if (lane == 0) {
          s_abort = 1;
          record_status(status, WINA_ERR_TIMEOUT);
        }
        break;
      }
      unsigned char* st = gbase + (size_t)s * stage_bytes;
      if (lane == 0) tc::mbar_arrive_expect_tx(&full[s], bytes);
      __syncwarp();
      if (row0 >= 0) {
        // 64 consecutive channels: one tile per 64-output box
        if (lane < 2) tc::tma_load_2d(st + (size_t)lane * (kUChunk * 128), &tmT, m0 + 64 * lane, row0, &full[s]);
      } else {
        // lane l gathers rows 4q .. 4q + 3 (q = l % 16) of output box l / 16
        const int q = lane & 15, box = lane >> 4;
        int rr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 4 * q + i;
          const int32_t a0 = __shfl_sync(0xffffffffu, u0, r & 31), a1 = __shfl_sync(0xffffffffu, u1, r & 31);
          rr[i] = r < 32 ? a0 : a1;
        }
        tc::tma_gather4(st + (size_t)box * (kUChunk * 128) + (size_t)q * 512, &tmA, m0 + 64 * box, rr[0], rr[1],
                        rr[2], rr[3], &full[s]);
      }
      if (lane < P) tc::tma_load_2d(st + a_bytes + (size_t)lane * x_bytes, &tmX, c * kUChunk, lane * NP, &full[s]);
      ++issued;
      row0 = nrow;
      u0 = n0;
      u1 = n1;
    }
    // let every copy issued land before the CTA can exit
    if (lane == 0) {
      for (int s = 0; s < S && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / S) * S;  // last iteration that used stage s
        tc::mbar_wait(&full[s], (uint32_t)((last / S) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, NP, 1);
      for (int c = c0; c < c1; ++c) {
        const int it = c - c0, s = it % S;
        if (!tc::mbar_wait(&full[s], (uint32_t)((it / S) & 1)) || *(volatile int*)&s_abort) {
          s_abort = 1;
          record_status(status, WINA_ERR_TIMEOUT);
          break;
        }
        tc::tc_fence_after();
        const uint32_t sa = sbase + (uint32_t)s * stage_bytes;
#pragma unroll
        for (int kk = 0; kk < kUChunk / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sa + (uint32_t)kk * 2048u, kUChunk * 128u, 1024u);
          for (int p = 0; p < P; ++p) {  // every part accumulates into the same D
            const uint64_t bd = tc::sw128_desc(sa + a_bytes + (uint32_t)p * x_bytes + (uint32_t)kk * 32u, 16u, 1024u);
            tc::mma_bf16(taddr, ad, bd, idesc, (it > 0 || kk > 0 || p > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(&done);
    }
  } else {
    // ---------------- D -> Y (warps 2-5, one lane quarter each) ----------------
    const int quarter = warp & 3;
    const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&done, 0u));
    tc::tc_fence_after();
    const int row = m0 + quarter * 32 + lane;
    if (ok && !*(volatile int*)&s_abort) {
      for (int c = 0; c < NP; c += 16) {
        uint32_t h[16];
        tc::tmem_ld16(taddr + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, h);
        tc::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int b = c + j;
          if (b < nb && row < m) atomicAdd(y + (int64_t)(b0 + b) * m + row, __uint_as_float(h[j]));
        }
      }
    } else if (!ok && lane == 0) {
      record_status(status, WINA_ERR_TIMEOUT);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc::tc_fence_after();
    tc::tmem_dealloc(taddr, ncols);
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------

namespace {
std::mutex g_tm_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::lock_guard<std::mutex> lk(g_tm_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

// bf16 matrix [rows][cols] (row stride cols), box [box_rows][box_cols], 128-byte swizzle.
static bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                           uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

UnionWs union_ws_layout(int64_t n, int64_t batch) {
  UnionWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = round_up(o + bytes, kAlign);
    return at;
  };
  const int64_t nblk = (n + kUChunk - 1) / kUChunk;
  w.kmax = (nblk + 1) * kUChunk;  // X~ columns: tile chunks plus packed gather chunks
  const int64_t nb = batch < kUBlock ? batch : kUBlock;
  w.np = (nb + 15) / 16 * 16;
  w.flag = take((size_t)n);
  w.chunk_row = take((size_t)(nblk + 1) * 4);
  w.slot = take((size_t)w.kmax * 4);
  w.pos = take((size_t)n * 4);
  w.info = take(16);
  w.xt = take((size_t)3 * w.np * w.kmax * 2);
  w.total = o;
  return w;
}

bool union_path_takes(int wdt, int64_t n, int64_t m, int64_t batch) {
  return wdt == WINA_BF16 && batch >= 2 && n <= 65536 && m >= 64 && m % 8 == 0 && device_sm_count() > 0;
}

wina_status_t launch_union_matvec(const void* Wt, int64_t n, int64_t m, const int32_t* idx, const float* xs, int k,
                                  const int32_t* count, int ld, int batch, float* y, void* ws, int32_t* status,
                                  cudaStream_t s, bool premarked) {
  const UnionWs L = union_ws_layout(n, batch);
  char* w = (char*)ws;
  uint8_t* flag = reinterpret_cast<uint8_t*>(w + L.flag);
  int32_t* chunk_row = reinterpret_cast<int32_t*>(w + L.chunk_row);
  int32_t* slot = reinterpret_cast<int32_t*>(w + L.slot);
  int32_t* pos = reinterpret_cast<int32_t*>(w + L.pos);
  uint32_t* info = reinterpret_cast<uint32_t*>(w + L.info);
  uint16_t* xt = reinterpret_cast<uint16_t*>(w + L.xt);
  CUtensorMap tmA, tmT, tmX;
  if (!encode_bf16_2d(&tmA, Wt, (uint64_t)m, (uint64_t)n, 64, 1)) return WINA_ERR_CUDA;
  if (!encode_bf16_2d(&tmT, Wt, (uint64_t)m, (uint64_t)n, 64, kUChunk)) return WINA_ERR_CUDA;
  if (!encode_bf16_2d(&tmX, xt, (uint64_t)L.kmax, (uint64_t)3 * L.np, 64, (uint32_t)L.np)) return WINA_ERR_CUDA;
  const int sms = device_sm_count();
  const int mtiles = (int)((m + 127) / 128);
  for (int b0 = 0; b0 < batch; b0 += kUBlock) {
    const int nb = std::min(kUBlock, batch - b0);
    const int NP = (nb + 15) / 16 * 16;
    if (NP != L.np) {  // the last, shorter block: its own box height
      if (!encode_bf16_2d(&tmX, xt, (uint64_t)L.kmax, (uint64_t)3 * NP, 64, (uint32_t)NP)) return WINA_ERR_CUDA;
    }
    // the union's flags: marked here from the lists, or already by the gate that made
    // them (one token block only)
    if (!(premarked && b0 == 0 && nb == batch)) k_union_mark<<<nb, 256, 0, s>>>(idx, ld, k, count, (int)n, b0, flag, status);
    k_union_plan<<<1, 1024, 0, s>>>(flag, (int)n, chunk_row, slot, pos, info);
    const int kcap = k >= 0 ? k : ld;
    const dim3 xgrid((unsigned)nb, (unsigned)std::max(1, (kcap + 255) / 256));
    k_union_xt<<<xgrid, 256, 0, s>>>(idx, xs, ld, k, count, (int)n, b0, NP, pos, info, xt, (int)L.kmax, y, (int)m);
    cudaError_t e;
    // pipeline depth: up to 8 stages; small token blocks keep the CTA under half an SM's
    // shared memory so that two CTAs share an SM
    const size_t stage_max = (size_t)2 * kUChunk * 128 + (size_t)3 * NP * 128;
    size_t smem = 1024 + (size_t)kUMaxStages * stage_max;
    const size_t cap = NP <= 64 ? (size_t)110 * 1024 : (size_t)226 * 1024;
    if (smem > cap) smem = cap;
    const int per_sm = NP <= 64 ? 2 : 1;
    // K splits: as many as keep every CTA of one wave resident
    int ksplit = std::max(1, sms * per_sm / mtiles);
    ksplit = (int)std::min<int64_t>(ksplit, L.kmax / kUChunk);
    e = ensure_smem_limit((const void*)k_union_gemm, smem);
    if (e != cudaSuccess) return cuda_status(e);
    k_union_gemm<<<mtiles * ksplit, kUT, smem, s>>>(tmA, tmT, tmX, chunk_row, slot, info, (int)m, nb, NP, ksplit, y,
                                                    b0, (int)smem, status);
    k_union_clear<<<xgrid, 256, 0, s>>>(idx, ld, k, count, (int)n, b0, NP, pos, xt, (int)L.kmax);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
  }
  return WINA_OK;
}

}  // namespace wina
