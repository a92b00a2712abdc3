"""CPU oracle of the NSNQuant hot path.  Test infrastructure only: the product
(CUDA library + binding) never imports it."""
