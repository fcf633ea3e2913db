// Test infrastructure: lets g++ compile the backward kernels' device source
// (chunked_gated_delta_14_b200/csrc/gdn_bwd_kernels.cuh) for the host, so a CPU
// test can run it block by block with one std::thread per CUDA thread.  It
// covers only what those kernels use: __global__/__device__ qualifiers,
// threadIdx/blockIdx, __syncthreads (a std::barrier over the block's threads),
// __shfl_xor_sync (an exchange buffer and a std::barrier per warp of 32 threads;
// the whole warp must call it together, as converged CUDA code does), dynamic
// shared memory (one host array, one block at a time), min, and the bit cast
// __uint_as_float.  The library never uses this file.
#pragma once
#include <algorithm>
#include <barrier>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

struct dim3h { unsigned x, y, z; };
struct float4 { float x, y, z, w; };
inline float4 make_float4(float x, float y, float z, float w) { return float4{x, y, z, w}; }
inline thread_local dim3h threadIdx;
inline dim3h blockIdx;
#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __shared__
inline std::barrier<> *g_block_barrier;
#define __syncthreads() g_block_barrier->arrive_and_wait()
inline std::barrier<> **g_warp_barriers;   // one per warp of the running block
inline float g_shfl_buf[1024];
inline float __shfl_xor_sync(unsigned, float v, int lane_mask) {
    const int t = (int)threadIdx.x;
    g_shfl_buf[t] = v;
    g_warp_barriers[t / 32]->arrive_and_wait();
    const float r = g_shfl_buf[(t & ~31) | ((t & 31) ^ lane_mask)];
    g_warp_barriers[t / 32]->arrive_and_wait();
    return r;
}
inline float __uint_as_float(unsigned u) { float f; std::memcpy(&f, &u, 4); return f; }
using std::min;
using std::max;
