"""B200-native verify + speculation-cache step of Speculative Speculative
Decoding (Saguaro).  The compute lives in libssd.so (CUDA, sm_100a); this
package is its thin ctypes binding (see ``binding``) plus the seeded workload
generator (``synth``)."""
