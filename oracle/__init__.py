"""CPU oracle for the BSFA prefill forward: test infrastructure only.

Only the tests, the smoke check and the bench's CPU-baseline leg may import this
package. The product path (the CUDA library and its Python binding) never does.
"""
