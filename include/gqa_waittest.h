/*
 * gqa_waittest.h -- the one extra entry point of libgqa_b200_waittest.so, a
 * build of the same sources as libgqa_b200.so made for testing the library's
 * failure handling.  Only the tests load it.
 *
 * In that build every internal wait of the kernels (a consumer waiting for
 * a tile, a producer waiting for a free ring slot) gives up after a
 * millisecond instead of about a second.  While the stall word set here is
 * non-zero, the producer of every kernel leaves its first stage unloaded, so
 * the waits on that stage run out: the kernel records GQA_ERR_TIMEOUT in the
 * device status word, lets the copies it did issue land, frees its tensor
 * memory and returns, and the context stays usable.  Every other entry point
 * of include/gqa.h is exported unchanged.
 *
 * The pages describe no such call: this exists only to exercise the bounded
 * waits.
 */
#ifndef GQA_B200_WAITTEST_H
#define GQA_B200_WAITTEST_H

#ifdef __cplusplus
extern "C" {
#endif

/* Sets (on != 0) or clears the stall word of the current device; returns
 * GQA_OK, or GQA_ERR_CUDA if the copy to the device fails.  Takes effect for
 * kernels launched after the copy completes. */
int gqa_test_set_stall(int on);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_WAITTEST_H */
