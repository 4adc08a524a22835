"""lossless_weight_compression_b200 -- libwcodec, a lossless BF16 weight codec for B200.

A block fixed-length code of BF16 exponents ("ENEC: A Lossless AI Model
Compression Method Enabling Fast Inference on Ascend NPUs", Abstract), written
for sm_100a: each BF16 word is split into its exponent byte and its
sign+mantissa byte; the mantissa bytes are stored raw and, within each block of
B elements, the exponents are stored as w-bit offsets from a per-block base.

The compute path is the C-ABI shared library ``libwcodec.so`` (hand-written
CUDA). ``wcodec`` is its ctypes binding; ``synth`` draws the seeded inputs.
Importing this package does not load the library; the first call into
``wcodec`` does, and fails loudly if it is missing.
"""
__all__ = ["wcodec", "synth"]
