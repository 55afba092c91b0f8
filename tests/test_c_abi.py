"""The boundary used from C: the public header compiles as strict C99 and a
C program links libfp8mlp.so with no Python or torch in the process.

On the CPU the program makes only calls that must fail their host-side
checks (so nothing reaches a GPU, wherever it runs).  On a B200 a second
program allocates its buffers with cudaMalloc, runs the calibration and
fp8mlp_mlp_train_step on the default stream, and writes its results to
files, which must equal the Python binding's results bit for bit."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "fp8_relu_mlp_b200")

HOST_PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include "fp8mlp.h"

int main(void) {
  uint16_t buf[64];
  void* fake = (void*)(((uintptr_t)buf + 15) & ~(uintptr_t)15); /* 16-byte aligned, never dereferenced */
  printf("version %s\n", fp8mlp_version());
  for (int c = 0; c <= 5; ++c) printf("code %d %s\n", c, fp8mlp_error_string(c));
  printf("count %d\n", fp8mlp_partial_amax_count(16384, 3072));
  /* a NULL input: rejected before anything is enqueued */
  int rc = fp8mlp_up_proj_fused(256, 64, 256, NULL, fake, fake, fake, fake, fake, NULL, 0, NULL);
  printf("up_null %d\n", rc);
  rc = fp8mlp_mlp_train_step(256, 64, 256, fake, NULL, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                             fake, fake, fake, fake, NULL);
  printf("step_null %d\n", rc);
  rc = fp8mlp_bwd_dx(128, 72, 256, fake, fake, fake, NULL);
  printf("dx_shape %d\n", rc);
  printf("detail %s\n", fp8mlp_last_error_detail());
  return 0;
}
"""

DEVICE_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <stdint.h>
#include <cuda_runtime.h>
#include "fp8mlp.h"

#define CK(x) do { int r_ = (int)(x); if (r_) { fprintf(stderr, "%s failed: %d (%s)\n", #x, r_, fp8mlp_last_error_detail()); return 1; } } while (0)

static void* load(const char* dir, const char* name, size_t bytes) {
  char path[1024];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  void* h = malloc(bytes);
  if (!f || fread(h, 1, bytes, f) != bytes) { fprintf(stderr, "cannot read %s\n", path); exit(1); }
  fclose(f);
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess || cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) exit(1);
  free(h);
  return d;
}

static int save(const char* dir, const char* name, const void* d, size_t bytes) {
  char path[1024];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  void* h = malloc(bytes);
  if (cudaMemcpy(h, d, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(h, 1, bytes, f) != bytes) return 1;
  fclose(f);
  free(h);
  return 0;
}

static void* zalloc(size_t bytes) {
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess || cudaMemset(d, 0, bytes) != cudaSuccess) exit(1);
  return d;
}

int main(int argc, char** argv) {
  if (argc != 5) return 2;
  const char* dir = argv[1];
  const int M = atoi(argv[2]), d = atoi(argv[3]), h = atoi(argv[4]);
  const size_t Md = (size_t)M * d, Mh = (size_t)M * h, hd = (size_t)h * d;
  uint16_t* x = (uint16_t*)load(dir, "x.bin", 2 * Md);
  uint16_t* W1 = (uint16_t*)load(dir, "W1.bin", 2 * hd);
  uint16_t* W2 = (uint16_t*)load(dir, "W2.bin", 2 * hd);
  uint16_t* dOut = (uint16_t*)load(dir, "dOut.bin", 2 * Md);
  const int npa = fp8mlp_partial_amax_count(M, h);
  uint8_t* W2q_t = (uint8_t*)zalloc(hd);
  float* w2inv = (float*)zalloc(16);
  fp8mlp_scale_state* st = (fp8mlp_scale_state*)zalloc(sizeof(fp8mlp_scale_state));
  uint16_t* post = (uint16_t*)zalloc(2 * Mh);
  uint8_t* q = (uint8_t*)zalloc(Mh);
  float* pa = (float*)zalloc(4 * (size_t)npa);
  uint16_t* out = (uint16_t*)zalloc(2 * Md);
  uint16_t* dPre = (uint16_t*)zalloc(2 * Mh);
  uint16_t* dX = (uint16_t*)zalloc(2 * Md);
  float* dW1 = (float*)zalloc(4 * hd);
  float* dW2 = (float*)zalloc(4 * hd);
  void* ws = zalloc(fp8mlp_workspace_size(M, d, h));
  CK(fp8mlp_scale_state_init(st, 2.0f, 1.0f, NULL));
  CK(fp8mlp_w2_fp8_cache_refresh(h, d, W2, W2q_t, w2inv, ws, NULL));
  /* step 0: calibration gives the first delayed scale */
  CK(fp8mlp_mlp_fwd(M, d, h, x, W1, NULL, NULL, NULL, st, post, NULL, pa, NULL, NULL, FP8MLP_FWD_CALIBRATE, NULL));
  CK(fp8mlp_amax_reduce_update_scale(pa, npa, st, NULL));
  for (int t = 0; t < 2; ++t)
    CK(fp8mlp_mlp_train_step(M, d, h, x, W1, W2, dOut, W2q_t, w2inv, st, post, q, pa, out, dPre, dX, dW1, dW2, ws,
                             NULL));
  unsigned int status = 0;
  CK(fp8mlp_get_device_status(&status, NULL));
  if (status) { fprintf(stderr, "device status %u\n", status); return 1; }
  CK(save(dir, "post.out", post, 2 * Mh) || save(dir, "q.out", q, Mh) || save(dir, "out.out", out, 2 * Md) ||
     save(dir, "dX.out", dX, 2 * Md) || save(dir, "dW1.out", dW1, 4 * hd) || save(dir, "dW2.out", dW2, 4 * hd) ||
     save(dir, "state.out", st, sizeof(fp8mlp_scale_state)) || save(dir, "W2q_t.out", W2q_t, hd));
  printf("ok\n");
  return 0;
}
"""


def _gcc():
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    return cc


def _build(tmp_path, src, name, cflags=(), libs=(), strict=True):
    """strict: ISO C99 with -pedantic (the library's header alone; the CUDA
    runtime's headers use extensions, so the device program is built
    without it)."""
    from fp8_relu_mlp_b200.build import build
    build()
    c = tmp_path / f"{name}.c"
    c.write_text(src)
    exe = tmp_path / name
    std = ["-std=c99", "-pedantic"] if strict else ["-std=gnu11"]
    cmd = [_gcc(), *std, "-Wall", "-Wextra", "-Werror", f"-I{INCLUDE}", *cflags, str(c), "-o",
           str(exe), f"-L{LIBDIR}", "-lfp8mlp", f"-Wl,-rpath,{LIBDIR}", *libs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_header_and_library_from_c(tmp_path):
    import torch
    exe = _build(tmp_path, HOST_PROGRAM, "host_calls")
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    lines = dict(l.split(" ", 1) for l in r.stdout.strip().splitlines() if not l.startswith("code"))
    assert "sm_100a" in lines["version"]
    assert lines["count"] == str(512 * 48)
    assert lines["up_null"] == "1" and lines["step_null"] == "1"   # FP8MLP_ERR_INVALID_ARG
    assert lines["dx_shape"] == "2"                                  # FP8MLP_ERR_UNSUPPORTED_SHAPE
    assert "multiples of 16" in lines["detail"]
    codes = [l for l in r.stdout.splitlines() if l.startswith("code")]
    assert codes[0] == "code 0 ok" and len(codes) == 6


@pytest.mark.gpu
def test_training_step_from_c_matches_the_binding(tmp_path):
    """A C program with its own cudaMalloc'd buffers and the default stream:
    calibration, then two fp8mlp_mlp_train_step calls; the same sequence
    through the Python binding gives the same bits."""
    import torch
    from fp8_relu_mlp_b200 import synth
    from fp8_relu_mlp_b200.block import MLPBlock
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = _build(tmp_path, DEVICE_PROGRAM, "device_step", cflags=(f"-I{cuda}/include",),
                 libs=(f"-L{cuda}/lib64", "-lcudart", f"-Wl,-rpath,{cuda}/lib64"), strict=False)
    M, d, h = 300, 128, 512
    P = synth.make_problem(M, d, h, seed=13)
    for k in ("x", "W1", "W2", "dOut"):
        (tmp_path / f"{k}.bin").write_bytes(np.ascontiguousarray(P[k]).tobytes())
    r = subprocess.run([str(exe), str(tmp_path), str(M), str(d), str(h)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
    b = MLPBlock(M, d, h)
    for k in ("x", "W1", "W2", "dOut"):
        getattr(b, k).copy_(MLPBlock.bits_to_bf16(P[k], b.device))
    b.refresh_w2_cache()
    b.calibrate()
    for _ in range(2):
        b.train_step_native()
    torch.cuda.synchronize()

    def host(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.uint8).numpy().tobytes()

    for name, t in (("post", b.post), ("q", b.post_fp8), ("out", b.out), ("dX", b.dX), ("dW1", b.dW1),
                    ("dW2", b.dW2), ("state", b.state), ("W2q_t", b.W2q_t)):
        assert (tmp_path / f"{name}.out").read_bytes() == host(t), name
