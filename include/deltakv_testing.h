/*
 * deltakv_testing.h -- test support of the DeltaKV library (libdeltakv.so).
 *
 * Not part of compression or decode.  The tensor-core kernels evaluate the
 * codec nonlinearity (GELU between the two layers of the compressor and of
 * the decompressor, "Processo di Compressione" step 4 and "Ricostruzione"
 * of the DeltaKV summary, section 3) with fast approximations of their own;
 * this entry point runs exactly those device functions on caller-chosen
 * inputs so that a test can hold them to their stated error bounds.
 */
#ifndef DELTAKV_TESTING_H
#define DELTAKV_TESTING_H

#include "deltakv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Device implementations of the nonlinearity that deltakv_test_activation
 * can run. */
typedef enum {
    DELTAKV_TEST_ACT_GELU_ERFF = 0,   /* x/2 (1 + erff(x / sqrt 2)), CUDA's erff, fp32 */
    DELTAKV_TEST_ACT_GELU_FAST = 1,   /* the fp32 polynomial form (compressor MLP) */
    DELTAKV_TEST_ACT_GELU_FAST2 = 2,  /* the same on two values at once (packed fp32x2) */
    DELTAKV_TEST_ACT_GELU_TANH = 3,   /* tanh form with CUDA's tanhf, fp32 */
    DELTAKV_TEST_ACT_GELU_TANHFIT2 = 4 /* the decode token loop's form: fitted tanh argument,
                                          MUFU tanh, packed fp32x2 (before its fp16 rounding) */
} deltakv_test_act_form;

/* y[i] = form(x[i]) for 0 <= i < n, computed on the device on `stream`.
 *   x, y : device float32 arrays of n elements (caller-owned; y written);
 *          the forms that work on pairs take x[2i], x[2i+1] together (an
 *          odd tail is paired with 0 and only its first result is kept).
 * Errors: INVALID_ARG (unknown form, n < 0, NULL pointer with n > 0),
 * CUDA (launch failed).  n == 0 launches nothing. */
deltakv_status deltakv_test_activation(int32_t form, const float* x, float* y, int64_t n,
                                       deltakv_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DELTAKV_TESTING_H */
