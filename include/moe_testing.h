/*
 * moe_testing.h -- test hooks of libmoe.so.  Not part of the layer's API;
 * they expose internal device functions so tests can check them alone.
 */
#ifndef MOE_TESTING_H
#define MOE_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* y[i] = the routing softmax's float32 exponential of x[i], computed by the
 * device function the router kernels use (Cody-Waite reduction, degree-7
 * Taylor polynomial in Horner form with fused multiply-adds, exact 2^n
 * scaling; +0 below -87).  x, y: device float32 arrays of n elements.
 * Returns a moe_status. */
int moe_test_exp_c(const float *x, float *y, int64_t n, void *stream);

/* Number of SMs the library sizes its persistent grids for on the current
 * device (0 if no device). */
int moe_test_num_sms(void);

/* Grouped GEMMs of the tensor-core path: single = 1 makes every later call
 * use the single-CTA kernels (k_gemm1, k_gemm2); 0 (the default) runs the
 * gate/up GEMM on the CTA-pair kernel (k_gemm1_pair) when I is a multiple
 * of 256 and the device holds at least one pair.  Process-wide, not
 * thread-safe; for tests and timing.  Returns a moe_status. */
int moe_test_set_grouped_single(int single);

/* CTA pairs of a pair GEMM the current device holds at once (the kernel's
 * grid is twice this): which 1, the gate/up GEMM (the one pair kernel); 0 if
 * it cannot be launched; -1 without a device or for another `which`. */
int moe_test_grouped_pairs(int which);

/* Set how long the library's bounded device waits (mbarrier phases,
 * cross-CTA flags, the grid barrier, the one-token layer's router exchange)
 * spin before they give up and record MOE_ERR_TIMEOUT, for the current
 * device, in nanoseconds (default 2e9).  Synchronous.  For tests that make a
 * wait run out; set it back afterwards.  Returns a moe_status. */
int moe_test_set_wait_limit_ns(uint64_t ns);

/* Launch one CTA that waits, with the library's bounded waits, on something
 * nothing ever completes: which 0, a flag in the workspace header; 1, an
 * mbarrier phase no thread arrives on; 2, the one-token layer's router
 * exchange for a tag no CTA publishes.  The wait gives up at the wait limit,
 * records MOE_ERR_TIMEOUT in the workspace's status word and the kernel
 * returns; the context stays usable.  Enqueued on `stream`.  Returns a
 * moe_status. */
int moe_test_wait_never_set(void *ws, size_t ws_bytes, int which, void *stream);

/* Re-run only the expert kernel of the last moe_layer call made with this
 * workspace, these shapes and these flags, reusing the logits (T == 1, where
 * the kernel routes the token itself) or the routing tables (T > 1) that call
 * left in the workspace: the single-pass decode kernel when flags carry
 * MOE_WDOWN_CHANNEL_MAJOR (its output accumulator is left as it ends; y is
 * not written), else the two-phase streaming kernel (writes y).  Launched
 * without programmatic dependent launch, so events recorded around it on
 * `stream` bracket this one kernel.  Used to time the dominant kernel alone.
 * Arguments as for moe_layer.  Returns a moe_status. */
int moe_test_expert_stream(const void *x_bf16, const void *w_gate_bf16, const void *w_up_bf16,
                           const void *w_down_bf16, int T, int d, int E, int I, int k1, int k2,
                           void *y, int y_dtype, int flags, void *ws, size_t ws_bytes,
                           void *stream);

/* The kernels of the grouped tensor-core expert FFN launched alone, without
 * programmatic dependent launch, on the routing tables a previous moe_layer
 * call left in `ws` (same shapes, k1).  `which` is a bit set: 4 copies the
 * routed tokens' x rows into expert order, 1 runs the gate/up GEMM with the
 * SwiGLU epilogue (writes h), 2 the down GEMM with the weighted combine (adds
 * into the workspace's float32 accumulator, whose contents are then
 * meaningless); 8 alone runs the down GEMM storing per-slot rows (the
 * moe_expert_ffn epilogue) over the gathered rows' space.  For timing the
 * kernels separately.  Shapes must satisfy the
 * grouped path (d and I multiples of 128).  Returns a moe_status. */
int moe_test_expert_grouped(const void *x_bf16, const void *w_gate_bf16, const void *w_up_bf16,
                            const void *w_down_bf16, int T, int d, int E, int I, int k1, int which,
                            void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_TESTING_H */
