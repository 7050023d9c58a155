// The input ring and the code-tile output shared by the TMA-fed quantisers.
//
// A persistent CTA visits the 128 x 128 tiles blockIdx.x, blockIdx.x +
// gridDim.x, ...; iteration `it` uses input stage it % STAGES and code tile
// it % CODE_BUFS.  Thread 0 keeps STAGES input tiles in flight with 2-D tensor
// copies (rows and columns past the matrix arrive as zeros) and writes each
// tile's codes back with one tensor store (which clips at the matrix edge), so
// the other threads touch global memory only for the scales.  Per iteration:
//   every thread   wait(it)                 the input tile has landed
//   thread 0       code_tile_free()         the store that last read this
//                                           iteration's code tile is done
//   CTA barrier    every thread holds its values
//   thread 0       refill(tile, it)         the stage takes the tile STAGES
//                                           iterations on
//   every thread   writes its codes, fence_proxy_async_smem()
//   CTA barrier, then thread 0 store(...)
// and after the loop thread 0 runs finish(ok, it).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "sm100.cuh"

namespace bsg {

template <int STAGES, int CODE_BUFS>
struct TileRing {
  static_assert(CODE_BUFS == 1 || CODE_BUFS == 2, "one or two code tiles");
  uint64_t* full;          // [STAGES] mbarriers: thread 0's arrival plus the copy's bytes
  volatile int* abort;     // CTA-wide flag raised by a wait that gave up
  const CUtensorMap* tmx;  // the input, in 128 x 128 boxes
  uint8_t* stages;         // input tile s at stages + s * stage_bytes
  uint32_t stage_bytes;
  long long ctiles, ntiles;  // column blocks, tiles

  // Thread 0, before the CTA-wide barrier that publishes the mbarriers.
  __device__ __forceinline__ void init(const CUtensorMap* tmq) const {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(tmx);
    tma_prefetch_desc(tmq);
  }

  __device__ __forceinline__ void issue(long long tile, int s) const {
    const long long rb = tile / ctiles, cb = tile - rb * ctiles;
    mbar_arrive_expect_tx(&full[s], stage_bytes);
    tma_load_3d(stages + static_cast<uint32_t>(s) * stage_bytes, tmx, &full[s], static_cast<int>(cb * 128),
                static_cast<int>(rb * 128), 0);
  }

  // Thread 0: the first STAGES tiles.
  __device__ __forceinline__ void start() const {
    for (int s = 0; s < STAGES; ++s) {
      const long long tile = blockIdx.x + static_cast<long long>(s) * gridDim.x;
      if (tile < ntiles) issue(tile, s);
    }
  }

  // Every thread: iteration it's tile is in shared memory; false once a wait
  // gave up (then the CTA winds down after the next barrier).
  __device__ __forceinline__ bool wait(int it, uint32_t* err) const {
    return wait_bounded(&full[it % STAGES], static_cast<uint32_t>(it / STAGES) & 1u, abort, err,
                        kErrTimeout | kRoleConsumer | kWaitStageFull);
  }

  // Thread 0: the tensor store issued CODE_BUFS iterations ago, the last to
  // read this iteration's code tile, has read it.
  __device__ __forceinline__ void code_tile_free() const {
    if constexpr (CODE_BUFS == 2) {
      bulk_wait_read1();
    } else {
      bulk_wait_read_all();
    }
  }

  // Thread 0, once every thread holds iteration it's values (`tile` is that
  // iteration's tile): the stage takes the tile STAGES iterations on.
  __device__ __forceinline__ void refill(long long tile, int it) const {
    const long long next = tile + static_cast<long long>(STAGES) * gridDim.x;
    if (next < ntiles) {
      fence_proxy_async_smem();  // the threads' reads of the stage, before the copy overwrites it
      issue(next, it % STAGES);
    }
  }

  // Thread 0, after every writer fenced its code-tile writes for the async
  // proxy and a CTA barrier: the code tile to (c0, c1) of `tmq`.
  __device__ __forceinline__ void store(const CUtensorMap* tmq, const void* codes, long long c0, long long c1) const {
    tma_store_3d(tmq, codes, static_cast<int>(c0), static_cast<int>(c1), 0);
    bulk_commit();
  }

  // Thread 0, after the loop (`it`: the iteration it ended at): every store is
  // complete, and after a wait that gave up the copies still in flight have
  // landed before the CTA retires.
  __device__ __forceinline__ void finish(bool ok, int it) const {
    bulk_wait_all();
    if (ok) return;
    volatile int never = 0;
    for (int j = it; j < it + STAGES; ++j) {
      const long long tile = blockIdx.x + static_cast<long long>(j) * gridDim.x;
      if (tile < ntiles) wait_bounded(&full[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u, &never, nullptr, 0);
    }
  }
};

}  // namespace bsg
