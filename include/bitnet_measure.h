/*
 * bitnet_measure.h - measurement and self-test entry points of libbitnet.so.
 *
 * These are not steps of the BitLinear method: they measure the hardware the
 * method's kernels run on, so that roofline fractions use a measured
 * denominator, and exercise the library's failure path.  Same conventions as bitnet.h (device pointers owned by the
 * caller, asynchronous on `stream`, host-side validation, bitnet_status codes).
 */
#ifndef BITNET_B200_MEASURE_H
#define BITNET_B200_MEASURE_H

#include <stdint.h>

#include "bitnet.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Dense int8 tensor-core throughput in the instruction form of the BitLinear
 * GEMM (tcgen05.mma.cta_group::1.kind::i8, A from tensor memory, B from shared
 * memory, int32 accumulators in tensor memory).  `ctas` CTAs (one per SM: each
 * holds all 512 tensor-memory columns) each issue n_mma MMAs of
 * 128 x bn x 32 back to back into one accumulator and wait for them.
 * cycles, nanos: out, [ctas] device arrays: SM clock cycles and globaltimer
 *                nanoseconds from the first issue to the last completion.
 * Integer operations: 2 * 128 * bn * 32 * n_mma per CTA.
 * Limits: bn 128 or 256; 1 <= n_mma <= 2^24; 1 <= ctas <= 4096.
 */
BITNET_API int bitnet_measure_i8_mma(int n_mma, int bn, int ctas, unsigned long long* cycles,
                                     unsigned long long* nanos, void* stream);

/*
 * Self-test of the failure path of the pipelines' bounded waits.  Enqueues one
 * kernel whose single thread waits on a barrier that nothing completes, with
 * the wait every kernel of the library uses: after about two seconds it gives
 * up, records a nonzero code in the device error flag (read it with
 * bitnet_device_error) and the kernel exits normally.  No fault, trap or
 * endless loop is involved; the CUDA context stays usable.
 */
BITNET_API int bitnet_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_MEASURE_H */
