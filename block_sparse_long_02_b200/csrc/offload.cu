// Host-offloaded K/V caches for decoding. A decode step reads only the
// selected blocks and the tail of each sequence ("QSA (Qwen Sparse Attention)"
// concept page, (B): attention restricted to the selected blocks' tokens), so
// the core K/V caches can live in host memory (pinned, mapped into the device
// address space) with an HBM cache of blocks in front of them, as the
// community KV-offloading port on the "QSA" knowledge page (kongchang) does:
// history in host memory, hot data and the indexer's caches on the GPU. The decode
// attention reads a block from its hot slot when the slot's tag names it and
// from host memory otherwise; this kernel then installs the step's missed
// blocks for the steps that follow.
//
// The hot cache is direct-mapped: block b may only sit in slot b % blocks (the
// extra tail slot after them is kept by the decode step's append). Of
// the selected blocks that share a slot, the lowest one is installed (the
// selection is ascending), so the cache contents are a deterministic function
// of the selections. Blocks before the current one never change once complete,
// so an installed copy stays valid.
#include <algorithm>

#include "kernels.h"

namespace qsa {
namespace {

constexpr int IT = 512;  // threads per CTA

__global__ void __launch_bounds__(IT) install_hot_kernel(const int64_t* __restrict__ pos, int64_t cap, int r,
                                                         int kB, int kv_heads, const int32_t* __restrict__ sel,
                                                         const int32_t* __restrict__ nsel,
                                                         const uint16_t* __restrict__ host_k,
                                                         const uint16_t* __restrict__ host_v,
                                                         uint16_t* __restrict__ hot_k, uint16_t* __restrict__ hot_v,
                                                         int32_t* __restrict__ tags, int32_t blocks) {
    __shared__ __align__(16) int32_t slot_of[kMaxKB];  // slot of entry k, -1 for an invalid entry
    __shared__ int32_t todo[kMaxKB];                   // first the entries' blocks, then the blocks to install
    __shared__ int n_todo;
    const int s = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // The selection was complete when the attention kernel before this one
    // passed its dependency wait (which it does before letting this kernel
    // launch), and the block slots' tags are written only by this kernel in
    // the previous step: so everything up to the copies overlaps the
    // attention. The copies
    // overwrite hot slots the attention reads and wait for it to finish.
    const int64_t p = pos[s];  // an input of the step
    if (p < 0 || p >= cap) {
        pdl_wait();
        pdl_trigger();
        return;
    }
    const int64_t cur = p / r;
    int ns = __ldcg(nsel + s);
    ns = ns < 0 ? 0 : (ns > kB ? kB : ns);
    const int ns4 = (ns + 3) & ~3;
    for (int k = tid; k < ns4; k += IT) {
        const int32_t b = k < ns ? __ldcg(sel + (size_t)s * kB + k) : -1;
        const bool ok = b >= 0 && (int64_t)b < cur;
        todo[k] = ok ? b : -1;
        slot_of[k] = ok ? b % blocks : -1;
    }
    if (tid == 0) n_todo = 0;
    __syncthreads();
    int32_t* tg = tags + (size_t)s * (blocks + 1);
    // Entries to install: the first entry of its slot (no lower entry has the
    // same slot) whose slot does not already hold its block.
    int32_t mine[kMaxKB / IT];
    int nmine = 0;
    for (int k = tid; k < ns; k += IT) {
        const int32_t b = todo[k], sl = slot_of[k];
        if (b < 0) continue;
        bool first = true;
        const int4* v4 = reinterpret_cast<const int4*>(slot_of);
        for (int j4 = 0; j4 < (k >> 2) && first; ++j4) {
            const int4 x = v4[j4];
            first = x.x != sl && x.y != sl && x.z != sl && x.w != sl;
        }
        for (int j = k & ~3; j < k && first; ++j) first = slot_of[j] != sl;
        if (first && __ldcg(tg + sl) != b) mine[nmine++] = b;
    }
    __syncthreads();  // every read of todo's first contents is done
    for (int e = 0; e < nmine; ++e) todo[atomicAdd(&n_todo, 1)] = mine[e];
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    // Copy each block (r tokens x kv_heads x 128 values, K and V) with one warp,
    // then publish it in the tag; the sequence's CTAs (which all found the
    // same list) take every gridDim.x-th block.
    const int n16 = r * kv_heads * kHeadDim / 8;  // 16-byte pieces per block and cache
    const size_t hot_seq = (size_t)s * (blocks + 1) * r * kv_heads * kHeadDim;
    const int wstride = (int)gridDim.x * (IT / 32);
    for (int e = (int)blockIdx.x * (IT / 32) + warp; e < n_todo; e += wstride) {
        const int32_t b = todo[e];
        const int32_t slot = b % blocks;
        const size_t src = ((size_t)s * cap + (size_t)b * r) * kv_heads * kHeadDim;
        const size_t dst = hot_seq + (size_t)slot * r * kv_heads * kHeadDim;
        const uint4* sk = reinterpret_cast<const uint4*>(host_k + src);
        const uint4* sv = reinterpret_cast<const uint4*>(host_v + src);
        uint4* dk = reinterpret_cast<uint4*>(hot_k + dst);
        uint4* dv = reinterpret_cast<uint4*>(hot_v + dst);
        int c = lane;
        for (; c + 96 < n16; c += 128) {  // four pieces of each cache in flight per lane
            uint4 a[4], b[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a[j] = sk[c + 32 * j];
                b[j] = sv[c + 32 * j];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                dk[c + 32 * j] = a[j];
                dv[c + 32 * j] = b[j];
            }
        }
        for (; c < n16; c += 32) {
            dk[c] = sk[c];
            dv[c] = sv[c];
        }
        __syncwarp();
        if (lane == 0) tg[slot] = b;
    }
}

}  // namespace

cudaError_t launch_install_hot(const LayerDims& L, int batch, const int64_t* pos, int64_t cap, const int32_t* sel,
                               const int32_t* nsel, const uint16_t* host_k, const uint16_t* host_v, uint16_t* hot_k,
                               uint16_t* hot_v, int32_t* tags, int64_t blocks, cudaStream_t st) {
    if (batch <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // CTAs per sequence: enough copying warps for a step where most blocks miss.
    const int x = std::max(1, std::min(8, sms / batch));
    note_launch();
    if (blocks < 1 || blocks >= INT32_MAX) return cudaErrorInvalidValue;
    return launch_pdl(install_hot_kernel, dim3((unsigned)x, (unsigned)batch), dim3(IT), 0, st, pos, cap, L.r, L.kB, L.kv_heads,
                      sel, nsel, host_k, host_v, hot_k, hot_v, tags, (int32_t)blocks);
}

}  // namespace qsa
