"""Write sampled oracle outputs of a full-size configuration.

The full 1080p decoder (8160 tokens, 16 blocks, W = 2) is too slow for the fp64
oracle to run inside a test, so this script runs it once, offline, on frames
0..3 (ring warm-up and the first wrap-around) and stores, per frame, the
values at 65536 seeded random pixel positions plus the output's L2 norm.
tests/test_gpu_fullsize.py regenerates the same seeded inputs, decodes them on
the GPU through the C ABI and compares at the stored positions.

Only oracle/ and fd_synth are used: no value here comes from the CUDA path.

    python tests/golden/make_fullsize_golden.py 1080p_wan22 4
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import fd_synth  # noqa: E402
import oracle  # noqa: E402

N_SAMPLES = 65536


def sample_positions(cfg, seed=12345):
    rng = np.random.default_rng(seed)
    size = int(np.prod(cfg.out_shape))
    return np.sort(rng.choice(size, size=N_SAMPLES, replace=False)).astype(np.int64)


def main(name="1080p_wan22", frames=4):
    cfg = fd_synth.CONFIGS[name]
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=frames)
    pos = sample_positions(cfg)
    dec = oracle.OracleDecoder(cfg, w)
    vals, norms = [], []
    for t in range(frames):
        t0 = time.time()
        y = dec.decode_frame(z[t]).reshape(-1)
        vals.append(y[pos])
        norms.append(float(np.linalg.norm(y)))
        print(f"frame {t}: {time.time() - t0:.1f} s, |y| = {norms[-1]:.6e}", flush=True)
    out = os.path.join(HERE, f"{name}_frames0-{frames - 1}.npz")
    np.savez_compressed(out, positions=pos, values=np.stack(vals), norms=np.array(norms),
                        config=name, frames=frames)
    print("wrote", out)


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else "1080p_wan22",
         int(sys.argv[2]) if len(sys.argv) > 2 else 4)
