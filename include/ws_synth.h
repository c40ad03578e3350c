/*
 * ws_synth.h -- seeded synthetic input generator on the device (libws_synth.so).
 *
 * Not part of the unit-step method: the tests and the benchmark use it to fill
 * large inputs (a 50 GB cache) directly in device memory.  It reproduces, bit
 * for bit, the numpy generator kv_cache_serving_ws_b200/synth.py:
 * element i of stream `key` is table_vals[#{k : table_thr[k] <= r}] with
 * r = top 32 bits of SplitMix64(key + (i + 1) * 0x9E3779B97F4A7C15).
 */
#ifndef WS_SYNTH_H
#define WS_SYNTH_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Fill dst[0 .. n) (device, bf16 patterns) with the elements index0 .. index0+n-1
 * of stream `key`.  table_thr (uint64, ascending) and table_vals (uint16) are
 * device copies of the generator's inverse-CDF table, 1..8192 entries.
 * Returns 0, -1 on a bad argument, -7 on a CUDA error.  Asynchronous on `stream`.
 */
int ws_synth_fill_normal_bf16(uint16_t* dst, int64_t n, uint64_t key, int64_t index0,
                              const uint64_t* table_thr, const uint16_t* table_vals, int32_t table_len,
                              cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WS_SYNTH_H */
